"""Build ``libmoe.so`` (all CUDA sources, sm_100a) in-tree next to this file.

    python -m load_balanced_dispatch_warp_b200.build [--force] [-v]

nvcc cross-compiles for sm_100a without a GPU.  Every ``csrc/*.cu`` file is compiled to
an object in parallel (``_build/``), then linked into one shared library.  The CUDA
runtime is linked statically and the driver API is reached through
cudaGetDriverEntryPoint, so the library loads on a machine without a GPU driver (its
calls then report an error).

The library is rebuilt whenever any ``csrc/*.cu``, ``csrc/*.cuh`` or ``include/*.h``
file is newer than it (found by glob, so a new header is watched without a list to keep).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmoe.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def dependencies():
    """Every file a build reads: the sources, the internal headers and the public ABI."""
    return (sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")))
            + sorted(glob.glob(os.path.join(INCLUDE, "*.h"))))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in dependencies())


def _compile_cmd(src: str, obj: str, verbose: bool):
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
           f"-I{INCLUDE}", f"-I{CSRC}", "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    objs, procs = [], []
    for src in sources():
        obj = os.path.join(OBJDIR, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        procs.append((src, subprocess.Popen(_compile_cmd(src, obj + ".tmp", verbose),
                                            stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                            text=True)))
    failed = False
    for src, p in procs:
        out, errtxt = p.communicate()
        if p.returncode != 0:
            failed = True
            sys.stderr.write(f"--- {os.path.basename(src)}\n{out}{errtxt}")
        elif verbose:
            sys.stderr.write(f"--- {os.path.basename(src)}\n{errtxt}")
    if failed:
        raise RuntimeError("nvcc failed building libmoe.so")
    for obj in objs:
        os.replace(obj + ".tmp", obj)
    link = [nvcc(), *ARCH, "--shared", "-cudart", "static", "-o", LIB + ".tmp", *objs]
    res = subprocess.run(link, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed linking libmoe.so")
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
