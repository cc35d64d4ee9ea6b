"""The in-tree build rebuilds libmoe.so when ANY source it reads changes (no GPU needed):
every csrc/*.cu, csrc/*.cuh and include/*.h, found by glob.  A stale library would ship
an old kernel to the GPU tests, so touching a header that only some sources include
(csrc/plan_body.cuh, the plan body shared by the plan and fused routing kernels) must
make the library out of date."""
import os
import shutil

from load_balanced_dispatch_warp_b200 import build


def test_every_source_and_header_is_a_dependency():
    deps = {os.path.relpath(p, build.ROOT) for p in build.dependencies()}
    pkg = "load_balanced_dispatch_warp_b200/csrc/"
    on_disk = {pkg + f for f in os.listdir(build.CSRC) if f.endswith((".cu", ".cuh"))}
    on_disk |= {"include/" + f for f in os.listdir(build.INCLUDE) if f.endswith(".h")}
    assert on_disk <= deps
    for must in ("plan_body.cuh", "common.cuh", "checks.cuh"):
        assert pkg + must in deps


def test_touching_a_header_makes_the_library_stale(tmp_path):
    lib = tmp_path / "libmoe.so"
    lib.write_bytes(b"")
    newest = max(os.path.getmtime(p) for p in build.dependencies())
    os.utime(lib, (newest + 10, newest + 10))
    assert build.up_to_date(str(lib))
    # a copy of the tree's dependency check against a header one second newer than lib
    header = os.path.join(build.CSRC, "plan_body.cuh")
    saved = tmp_path / "plan_body.cuh.saved"
    shutil.copy2(header, saved)
    try:
        os.utime(header, (newest + 20, newest + 20))
        assert not build.up_to_date(str(lib))
    finally:
        st = os.stat(saved)
        os.utime(header, (st.st_atime, st.st_mtime))
    assert build.up_to_date(str(lib))
