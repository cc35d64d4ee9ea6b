"""The C-ABI library loads, exports every entry point include/moe.h declares, and its
host-side checks answer without touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return M.lib()


def declared_functions():
    text = open(HEADER).read()
    return set(re.findall(r"^(?:int|int64_t|const char\*)\s+(moe_\w+)\s*\(", text, flags=re.M))


def test_header_declares_the_path(lib):
    names = declared_functions()
    assert set(M.ENTRY_POINTS) <= names
    assert set(M.HELPERS) <= names
    assert set(M.VARIANTS) <= names
    assert set(M.FUSED) <= names
    assert set(M.BACKWARD) <= names
    assert set(M.EXPERT_PARALLEL) <= names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_plan_layout_is_consistent(lib):
    E, R, S = 256, 32, 4
    L = M.plan_layout(E, R, S)
    B = E // R
    assert L.max_groups_per_rank == B + S
    assert L.room_prefix == L.kept_rows + R
    assert L.expert_home_off == L.room_prefix + R + 1
    assert L.stream_off == L.expert_home_off + E
    assert L.replica_expert == L.stream_off + E + 1
    assert L.replica_list == L.replica_expert + R * S
    assert L.n_groups == L.replica_list + 1 + R * S
    assert L.groups % 4 == 0 and L.groups >= L.n_groups + R
    assert L.words == L.groups + R * (B + S) * 4
    # per 256-token tile: a status word, its expert counts and its inclusive prefix, after
    # four header words (the status block padded to a multiple of 4 words)
    assert M.dispatch_workspace_words(16384, 256) == 68 + 2 * 64 * 256
    assert M.dispatch_workspace_words(257, 8) == 8 + 2 * 2 * 8
    assert M.dispatch_workspace_words(0, 8) == 4
    # the fixed-capacity rows: ceil(A / E * cf), the pages' fixture gives 5
    assert M.capacity_rows(16, 2, 8, 5, 4) == 5
    assert M.capacity_rows(16384, 8, 256, 1, 1) == 512
    assert M.capacity_rows(16384, 8, 256, 5, 4) == 640
    assert M.capacity_rows(0, 8, 256, 5, 4) == 0


def test_host_checks_reject_bad_arguments(lib):
    P = ctypes.c_void_p
    fake = P(4096)  # never dereferenced: every call below fails its host checks first
    # null error word
    assert lib.moe_topk(fake, 4, 8, 2, fake, fake, None, None) == M.MOE_ERR_ARG
    # k > E, E > 1024
    assert lib.moe_topk(fake, 4, 8, 9, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_topk(fake, 4, 2048, 2, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    # E % R != 0
    assert lib.moe_histogram_maxvio(fake, 4, 2, 8, 3, None, fake, fake, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    # T*k % R != 0
    assert lib.moe_plan_balanced(fake, 3, 1, 8, 2, 2, fake, fake, None) == M.MOE_ERR_SHAPE
    # too many group slots
    assert lib.moe_plan_balanced(fake, 4096, 1, 1024, 1024, 4, fake, fake, None) == M.MOE_ERR_SHAPE
    # d % 128 != 0
    assert lib.moe_dispatch(fake, fake, fake, 4, 2, 8, 4, 2, 96, fake, fake, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    # misaligned token rows
    assert lib.moe_dispatch(P(4098), fake, fake, 4, 2, 8, 4, 2, 128, fake, fake, fake, fake, fake, None) == M.MOE_ERR_ARG
    # F % 128 != 0, missing pool
    assert lib.moe_grouped_ffn(fake, fake, fake, fake, fake, fake, fake, fake, 4, 2, 8, 4, 2, 128, 200,
                               fake, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_grouped_ffn(fake, fake, fake, fake, fake, None, None, None, 4, 2, 8, 4, 2, 128, 256,
                               fake, fake, fake, None) == M.MOE_ERR_ARG
    assert lib.moe_combine(fake, fake, fake, 4, 33, 128, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_prefetch_replicas(fake, fake, fake, fake, 8, 4, 2, 128, 256, None, None, None, fake, None) == M.MOE_ERR_ARG
    assert lib.moe_status_string(M.MOE_ERR_SHAPE) == b"size limit violated"


def test_fused_dispatch_host_checks(lib):
    P = ctypes.c_void_p
    fake = P(4096)
    # index-only dispatch: null outputs, T*k % R != 0, E % R != 0
    assert lib.moe_dispatch_index(fake, fake, 4, 2, 8, 4, 2, fake, fake, None, fake, None) == M.MOE_ERR_ARG
    assert lib.moe_dispatch_index(fake, fake, 3, 1, 8, 2, 2, fake, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_dispatch_index(fake, fake, 4, 2, 8, 3, 2, fake, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    # gathered FFN: null x or src, F % 128 != 0, misaligned x, missing pool
    args = [fake, fake, fake, fake, fake, fake, fake, fake, fake, 4, 2, 8, 4, 2, 128, 256, fake, fake, fake, None]
    bad = list(args); bad[0] = None
    assert lib.moe_grouped_ffn_gather(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[1] = None
    assert lib.moe_grouped_ffn_gather(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[15] = 200
    assert lib.moe_grouped_ffn_gather(*bad) == M.MOE_ERR_SHAPE
    bad = list(args); bad[0] = P(4098)
    assert lib.moe_grouped_ffn_gather(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[6] = None
    assert lib.moe_grouped_ffn_gather(*bad) == M.MOE_ERR_ARG


def test_backward_host_checks(lib):
    P = ctypes.c_void_p
    fake = P(4096)
    assert lib.moe_combine_backward(fake, fake, fake, fake, 4, 2, 128, fake, fake, None, None) == M.MOE_ERR_ARG
    assert lib.moe_combine_backward(fake, fake, fake, fake, 4, 33, 128, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_dispatch_backward(fake, fake, 4, 2, 96, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_topk_backward(fake, fake, fake, 4, 8, 9, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_ffn_backward_workspace_bytes(4, 2, 8, 3, 2, 128, 256) == -1  # E % R
    n = lib.moe_ffn_backward_workspace_bytes(4096, 6, 64, 8, 8, 2048, 1408)
    assert n > 0 and n % 256 == 0
    args = [fake, fake, fake, fake, fake, fake, fake, 4, 2, 8, 4, 2, 128, 256, fake, fake, fake, fake,
            fake, 1 << 30, fake, None]
    bad = list(args); bad[15] = None  # dW1 missing
    assert lib.moe_grouped_ffn_backward(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[18] = P(4096 + 16)  # workspace not 256-byte aligned
    assert lib.moe_grouped_ffn_backward(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[19] = 1024  # workspace too small
    assert lib.moe_grouped_ffn_backward(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[13] = 200  # F % 128
    assert lib.moe_grouped_ffn_backward(*bad) == M.MOE_ERR_SHAPE


def test_ffn_tile_mode_switch(lib):
    """The tile-mode switch is host state only: checked, returns the previous mode."""
    prev = lib.moe_ffn_tile_mode()
    assert prev in (0, 1)
    assert lib.moe_set_ffn_tile_mode(2) == M.MOE_ERR_ARG
    assert lib.moe_set_ffn_tile_mode(-1) == M.MOE_ERR_ARG
    assert lib.moe_ffn_tile_mode() == prev
    assert lib.moe_set_ffn_tile_mode(1 - prev) == M.MOE_OK
    assert lib.moe_ffn_tile_mode() == 1 - prev
    assert M.set_ffn_tile_mode(prev) == 1 - prev
    assert lib.moe_ffn_tile_mode() == prev
    with pytest.raises(M.MoEError):
        M.set_ffn_tile_mode(2)
    assert lib.moe_ffn_tile_mode() == prev


def test_route_plan_host_checks(lib):
    """moe_route_plan answers bad arguments on the host, as its three separate calls do."""
    P = ctypes.c_void_p
    fake = P(4096)
    # logits, bias, T, E, k, R, S, idx, gate, counts, loads, maxvio, bal, plan, ws, err, stream
    args = [fake, None, 16, 8, 2, 4, 2, fake, fake, fake, fake, fake, fake, fake, fake, fake, None]
    for i in (0, 7, 8, 9, 10, 11, 12, 13, 14, 15):  # null logits / outputs / workspace / err
        bad = list(args); bad[i] = None
        assert lib.moe_route_plan(*bad) == M.MOE_ERR_ARG, i
    bad = list(args); bad[2] = 15  # T*k % R != 0
    assert lib.moe_route_plan(*bad) == M.MOE_ERR_SHAPE
    bad = list(args); bad[5] = 3  # E % R != 0
    assert lib.moe_route_plan(*bad) == M.MOE_ERR_SHAPE
    bad = list(args); bad[4] = 9  # k > E
    assert lib.moe_route_plan(*bad) == M.MOE_ERR_SHAPE
    bad = list(args); bad[3] = 2048; bad[5] = 8  # E > 1024
    assert lib.moe_route_plan(*bad) == M.MOE_ERR_SHAPE
    bad = list(args); bad[2] = 0; bad[0] = None; bad[7] = None; bad[8] = None  # T = 0: no rows
    # (accepted on the host; a launch would follow, so only the null-output case is probed)
    bad[9] = None
    assert lib.moe_route_plan(*bad) == M.MOE_ERR_ARG
    assert lib.moe_route_plan_workspace_words(64) == 16 * 64 + 1
    assert lib.moe_route_plan_workspace_words(0) == -1
    assert lib.moe_route_plan_workspace_words(1025) == -1


def test_fixed_capacity_and_fused_combine_host_checks(lib):
    """Host argument rules of the fixed-capacity calls and the fused combine (nothing is
    enqueued: every call below fails before any device work)."""
    P = ctypes.c_void_p
    fake = P(4096)
    assert lib.moe_capacity_rows(16, 2, 8, 0, 4) == -1
    assert lib.moe_capacity_rows(-1, 2, 8, 5, 4) == -1
    # dispatch_capacity: null counts, negative cap, d % 128, misaligned recv, E*cap*d too big
    base = [fake, fake, fake, 16, 2, 8, 5, 128, fake, fake, fake, fake, fake, None]
    bad = list(base); bad[2] = None
    assert lib.moe_dispatch_capacity(*bad) == M.MOE_ERR_ARG
    bad = list(base); bad[6] = -1
    assert lib.moe_dispatch_capacity(*bad) == M.MOE_ERR_ARG
    bad = list(base); bad[7] = 96
    assert lib.moe_dispatch_capacity(*bad) == M.MOE_ERR_SHAPE
    bad = list(base); bad[9] = P(4100)
    assert lib.moe_dispatch_capacity(*bad) == M.MOE_ERR_ARG
    bad = list(base); bad[6] = 1 << 20; bad[5] = 1024; bad[7] = 4096
    assert lib.moe_dispatch_capacity(*bad) == M.MOE_ERR_SHAPE
    # grouped_ffn_capacity: E > 1024, F % 128, rows * F too big
    assert lib.moe_grouped_ffn_capacity(fake, fake, fake, fake, 2048, 4, 128, 128, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_grouped_ffn_capacity(fake, fake, fake, fake, 8, 4, 128, 200, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_grouped_ffn_capacity(fake, fake, fake, fake, 1024, 1 << 20, 128, 4096, fake, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_grouped_ffn_capacity(fake, fake, fake, fake, 8, 4, 128, 128, fake, fake, None, None) == M.MOE_ERR_ARG
    # combine_capacity: k > 32, null gate
    assert lib.moe_combine_capacity(fake, fake, fake, 4, 33, 128, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_combine_capacity(fake, fake, None, 4, 2, 128, fake, fake, None) == M.MOE_ERR_ARG
    # fused combine: null out32 or perm, T*k % R != 0, misaligned out32, missing pool
    args = [fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, 4, 2, 8, 4, 2, 128, 256,
            fake, fake, fake, fake, None]
    bad = list(args); bad[19] = None
    assert lib.moe_grouped_ffn_combine(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[9] = None
    assert lib.moe_grouped_ffn_combine(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[11] = 3; bad[12] = 1
    assert lib.moe_grouped_ffn_combine(*bad) == M.MOE_ERR_SHAPE
    bad = list(args); bad[19] = P(4100)
    assert lib.moe_grouped_ffn_combine(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[5] = None
    assert lib.moe_grouped_ffn_combine(*bad) == M.MOE_ERR_ARG


def test_expert_parallel_host_checks(lib):
    """Host argument rules of the expert-parallel calls and the IPC helpers (nothing is
    enqueued: every call below fails before any device work)."""
    P = ctypes.c_void_p
    fake = P(4096)

    def table(n, addr=4096):
        return (ctypes.c_void_p * n)(*([addr] * n))

    # counts: null send, k > E
    assert lib.moe_ep_counts(fake, 4, 2, 8, fake, None, None) == M.MOE_ERR_ARG
    assert lib.moe_ep_counts(fake, 4, 9, 8, fake, fake, None) == M.MOE_ERR_SHAPE
    # plan: me outside [0, W), W > 64, E % W, too many groups
    plan_args = [fake, 2, 0, 16, 2, 8, 2, fake, fake, fake, fake, fake, fake, fake, None]
    bad = list(plan_args); bad[2] = 2
    assert lib.moe_ep_plan(*bad) == M.MOE_ERR_ARG
    bad = list(plan_args); bad[1] = 65; bad[5] = 1040
    assert lib.moe_ep_plan(*bad) == M.MOE_ERR_SHAPE
    bad = list(plan_args); bad[1] = 3
    assert lib.moe_ep_plan(*bad) == M.MOE_ERR_SHAPE
    bad = list(plan_args); bad[6] = 5000
    assert lib.moe_ep_plan(*bad) == M.MOE_ERR_SHAPE
    bad = list(plan_args); bad[12] = None
    assert lib.moe_ep_plan(*bad) == M.MOE_ERR_ARG
    # dispatch: a null or misaligned entry in the receive table, W*T*k too big
    disp = [fake, fake, fake, fake, 2, 16, 2, 8, 2, 128, fake, table(2), fake, fake, None]
    assert lib.moe_ep_dispatch(*disp[:11], table(2, 0), *disp[12:]) == M.MOE_ERR_ARG
    assert lib.moe_ep_dispatch(*disp[:11], table(2, 4100), *disp[12:]) == M.MOE_ERR_ARG
    bad = list(disp); bad[4] = 64; bad[5] = 1 << 24; bad[7] = 64
    assert lib.moe_ep_dispatch(*bad) == M.MOE_ERR_SHAPE
    bad = list(disp); bad[2] = None
    assert lib.moe_ep_dispatch(*bad) == M.MOE_ERR_ARG
    # prefetch: a short weight table is the caller's contract, a null entry is caught
    pre = [fake, table(2), table(2), table(2), 2, 1, 8, 2, 128, 256, fake, fake, fake, fake, None]
    bad = list(pre); bad[2] = table(2, 0)
    assert lib.moe_ep_prefetch(*bad) == M.MOE_ERR_ARG
    bad = list(pre); bad[9] = 200
    assert lib.moe_ep_prefetch(*bad) == M.MOE_ERR_SHAPE
    # grouped FFN: null group scratch, misaligned h
    ffn = [fake, fake, 2, 1, fake, fake, fake, fake, fake, fake, 16, 2, 8, 2, 128, 256, fake, fake,
           fake, fake, None]
    bad = list(ffn); bad[16] = None
    assert lib.moe_ep_grouped_ffn(*bad) == M.MOE_ERR_ARG
    bad = list(ffn); bad[17] = P(4098)
    assert lib.moe_ep_grouped_ffn(*bad) == M.MOE_ERR_ARG
    # combine: W = 0, k > 32, null table entry
    assert lib.moe_ep_combine(table(2), fake, fake, 0, 16, 2, 128, fake, fake, None) == M.MOE_ERR_ARG
    assert lib.moe_ep_combine(table(2), fake, fake, 2, 16, 33, 128, fake, fake, None) == M.MOE_ERR_SHAPE
    assert lib.moe_ep_combine(table(2, 0), fake, fake, 2, 16, 2, 128, fake, fake, None) == M.MOE_ERR_ARG
    # IPC helpers: null arguments; a host address is not a device allocation
    off = ctypes.c_int64(0)
    h = ctypes.create_string_buffer(M.IPC_HANDLE_BYTES)
    assert lib.moe_ipc_export(None, h, ctypes.byref(off)) == M.MOE_ERR_ARG
    assert lib.moe_ipc_import(h, -1, ctypes.byref(P()), ctypes.byref(P())) == M.MOE_ERR_ARG
    assert lib.moe_ipc_close(None) == M.MOE_ERR_ARG


def test_expert_parallel_backward_host_checks(lib):
    """Host argument rules of the expert-parallel backward calls (nothing is enqueued)."""
    P = ctypes.c_void_p
    fake = P(4096)

    def table(n, addr=4096):
        return (ctypes.c_void_p * n)(*([addr] * n))

    assert lib.moe_ep_combine_backward(fake, table(2), fake, fake, 2, 16, 2, 128, table(2), None,
                                       fake, None) == M.MOE_ERR_ARG  # dgate missing
    assert lib.moe_ep_combine_backward(fake, table(2), fake, fake, 2, 16, 2, 128, table(2, 0), fake,
                                       fake, None) == M.MOE_ERR_ARG  # null dy entry
    assert lib.moe_ep_ffn_backward_workspace_bytes(16, 2, 8, 3, 2, 128, 256) == -1  # E % W
    assert lib.moe_ep_ffn_backward_workspace_bytes(16, 2, 1024, 1, 8, 128, 256) == -1  # B+S > 1024
    n = lib.moe_ep_ffn_backward_workspace_bytes(512, 6, 64, 8, 8, 2048, 1408)
    assert n > 0 and n % 256 == 0
    args = [fake, fake, fake, 2, 1, fake, fake, fake, fake, fake, fake, 16, 2, 8, 2, 128, 256,
            fake, fake, fake, fake, fake, P(4096 * 64), 1 << 30, fake, None]
    bad = list(args); bad[19] = None  # dP3 missing
    assert lib.moe_ep_grouped_ffn_backward(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[23] = 1024  # workspace too small
    assert lib.moe_ep_grouped_ffn_backward(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[22] = P(4096 + 16)  # workspace not 256-byte aligned
    assert lib.moe_ep_grouped_ffn_backward(*bad) == M.MOE_ERR_ARG
    bad = list(args); bad[4] = 2  # me outside [0, W)
    assert lib.moe_ep_grouped_ffn_backward(*bad) == M.MOE_ERR_ARG
    assert lib.moe_ep_reduce_home(fake, table(2), table(2, 0), table(2), 2, 0, 8, 2, 128, 256,
                                  fake, None) == M.MOE_ERR_ARG
    assert lib.moe_ep_dispatch_backward(table(2), fake, 2, 16, 2, 96, fake, fake, None) == M.MOE_ERR_SHAPE


def test_w2_conversion_host_checks(lib):
    P = ctypes.c_void_p
    fake = P(4096)
    assert lib.moe_w2_to_f16(fake, 12, fake, None) == M.MOE_ERR_SHAPE  # n % 8
    assert lib.moe_w2_to_f16(fake, -8, fake, None) == M.MOE_ERR_ARG
    assert lib.moe_w2_to_f16(None, 8, fake, None) == M.MOE_ERR_ARG
    assert lib.moe_w2_to_f16(P(4098), 8, fake, None) == M.MOE_ERR_ARG  # misaligned
    assert lib.moe_w2_to_f16(None, 0, None, None) == M.MOE_OK  # nothing to convert
