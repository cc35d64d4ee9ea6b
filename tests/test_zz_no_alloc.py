"""moe_dispatch_noalloc against moe_dispatch (needs a B200).

The no-allocation entry point serves callers that cannot allocate device memory when
they dispatch (an operator interface that hands over only inputs and outputs, or a hot
path that must not call cudaMalloc).  It must place every assignment exactly as
moe_dispatch does with a caller workspace: perm, src and the received rows bit for bit,
on two calls in a row with different traces (the shared static scratch keeps the first
call's contents when the second one runs).  Kept in a file of its own, collected last.
"""
import ctypes

import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    L = M.lib()
    f = L.moe_dispatch_noalloc
    P, Ii = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, Ii, Ii, Ii, Ii, Ii, Ii, P, P, P, P, P]
    f.restype = ctypes.c_int
    return L


def _routed(w):
    """Top-k, histogram and plan of a workload through the regular entry points."""
    layer = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, 128)
    logits = I.make_logits(w).cuda()
    x = I.make_x(w).cuda()
    layer.route(logits)
    layer.measure()
    layer.balance()
    torch.cuda.synchronize()
    assert int(layer.err.item()) == 0
    return layer, x


def _noalloc(lib, layer, x, w):
    recv = torch.full((w.A, w.d), -1.0, dtype=torch.bfloat16, device="cuda")
    perm = torch.full((w.T, w.k), -1, dtype=torch.int32, device="cuda")
    src = torch.full((w.A,), -1, dtype=torch.int32, device="cuda")
    err = layer.err.clone()
    st = lib.moe_dispatch_noalloc(x.data_ptr(), layer.idx.data_ptr(), layer.plan.data_ptr(), w.T,
                                  w.k, w.E, w.R, w.S, w.d, recv.data_ptr(), perm.data_ptr(),
                                  src.data_ptr(), err.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    assert st == M.MOE_OK
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return recv, perm, src


def test_noalloc_matches_dispatch_two_calls(lib):
    cases = [I.WORKLOADS["qwen_mv5"], I.small_workload("ragged", 300, 16, 4, 4, 2, 256, 128, alpha=1.0, seed=1)]
    for w in cases:  # two calls in a row, different traces and sizes
        layer, x = _routed(w)
        layer.dispatch(x)  # the regular entry point, with the caller's workspace
        torch.cuda.synchronize()
        recv, perm, src = _noalloc(lib, layer, x, w)
        assert torch.equal(perm, layer.perm)
        assert torch.equal(src, layer.src)
        assert torch.equal(recv, layer.recv)


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    fake = ctypes.c_void_p(4096)  # never dereferenced: the size check fails first
    T, E = 65536, 1024
    assert M.dispatch_workspace_words(T, E) > M.NOALLOC_SCRATCH_WORDS
    st = lib.moe_dispatch_noalloc(fake, fake, fake, T, 8, E, 8, 4, 128, fake, fake, fake, fake, None)
    assert st == M.MOE_ERR_SHAPE
    assert M.dispatch_workspace_words(65536, 512) <= M.NOALLOC_SCRATCH_WORDS
    assert M.dispatch_workspace_words(32768, 1024) <= M.NOALLOC_SCRATCH_WORDS
