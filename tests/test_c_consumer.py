"""The boundary is a C ABI: a plain C99 program (tests/abi_consumer.c) compiles against
include/moe.h with gcc -std=c99 -pedantic, links libmoe.so, and gets the same host-side
answers as the Python binding (CPU only; no call in it reaches a GPU)."""
import os
import shutil
import subprocess

import pytest

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("needs gcc")
    build.build()
    lib_dir = os.path.dirname(M.LIB_PATH)
    exe = str(tmp_path_factory.mktemp("c") / "consumer")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(HERE, "abi_consumer.c"),
           "-L", lib_dir, "-lmoe", f"-Wl,-rpath,{lib_dir}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60).stdout
    return dict(line.split(" ", 1) for line in out.strip().splitlines())


def test_layout_and_workspaces_match_the_binding(results):
    lay = M.plan_layout(64, 8, 8)
    assert int(results["layout_status"]) == M.MOE_OK
    assert int(results["layout_words"]) == lay.words
    assert int(results["layout_groups"]) == lay.groups
    assert int(results["layout_max_groups_per_rank"]) == lay.max_groups_per_rank == 8 + 8
    assert int(results["dispatch_workspace_words"]) == M.dispatch_workspace_words(4096, 64)
    assert int(results["route_plan_workspace_words"]) == M.route_plan_workspace_words(64)
    assert int(results["route_plan_workspace_words_bad"]) == -1


def test_host_checks_from_c(results):
    assert int(results["ffn_tile_mode"]) == 0
    assert int(results["set_ffn_tile_mode_bad"]) == M.MOE_ERR_ARG
    assert int(results["topk_null_logits"]) == M.MOE_ERR_ARG
    assert int(results["topk_k_above_E"]) == M.MOE_ERR_SHAPE
    assert int(results["plan_rows_not_divisible"]) == M.MOE_ERR_SHAPE
    assert int(results["route_plan_null_workspace"]) == M.MOE_ERR_ARG
    assert results["status_ok_string"] == M.lib().moe_status_string(M.MOE_OK).decode()
    assert (int(results["status_arg"]), int(results["status_shape"])) == (M.MOE_ERR_ARG, M.MOE_ERR_SHAPE)
