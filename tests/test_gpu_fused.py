"""Fused dispatch (needs a B200): moe_dispatch_index + moe_grouped_ffn_gather.

GEMM 1 gathers its rows as x[src[row]] instead of reading the dispatched copies, so every
output must equal the unfused path's bit for bit (same operand values, same MMA order), and
the layer must pass the same oracle checks: integer outputs bit-exact, h / y / out within
1e-2 * max(1, |oracle|).
"""
import numpy as np
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I
from load_balanced_dispatch_warp_b200.pipeline import HostPipeline

from harness import (check_ffn_combine_full, check_ffn_combine_sampled, check_integer_parity,
                     make_inputs, oracle_integer_path, run_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    M.lib()


def assert_same_outputs(Lf, Lu):
    assert torch.equal(Lf.perm, Lu.perm), "perm"
    assert torch.equal(Lf.src, Lu.src), "src"
    assert torch.equal(Lf.h, Lu.h), "h"
    assert torch.equal(Lf.y, Lu.y), "y"
    assert torch.equal(Lf.out, Lu.out), "out"


SMALL = [
    I.WORKLOADS["tiny"],
    # ragged groups: many partial 128-row tiles, rows past a group's end zero-filled
    I.small_workload("ragged", 300, 16, 4, 4, 2, 256, 384, alpha=1.0, seed=1),
    I.small_workload("mid", 1000, 64, 6, 8, 8, 512, 256, alpha=0.6, seed=2),
    I.small_workload("k1_d384", 96, 32, 1, 8, 2, 384, 128, alpha=1.5, seed=4),
    I.small_workload("one_rank", 64, 16, 4, 1, 0, 128, 128, alpha=1.0, seed=5),
    I.small_workload("hot", 512, 32, 4, 8, 4, 128, 256, alpha=2.5, seed=7),
    I.small_workload("wide_E", 200, 512, 8, 16, 12, 128, 128, alpha=0.3, seed=8),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_fused_layer_parity_small(w):
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    Lf = run_gpu(w, logits, x, weights, fused=True)
    Lu = run_gpu(w, logits, x, weights)
    if ref["err"]:
        assert int(Lf.err.item()) == ref["err"]
        return
    assert Lf.recv is None
    check_integer_parity(Lf, w, ref)
    check_ffn_combine_full(Lf, w, x, weights, ref)
    assert_same_outputs(Lf, Lu)


@pytest.mark.parametrize("name", ["near_balanced", "qwen_mv15", "mixtral", "deepseek"])
def test_fused_equals_unfused_full_size(name):
    w = I.WORKLOADS[name]
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    Lf = run_gpu(w, logits, x, weights, fused=True)
    assert int(Lf.err.item()) == 0
    check_integer_parity(Lf, w, ref)
    rng = np.random.default_rng(17)
    tokens = sorted(rng.choice(w.T, size=6, replace=False).tolist()) + [w.T - 1]
    check_ffn_combine_sampled(Lf, w, x, weights, ref, tokens)
    Lu = run_gpu(w, logits, x, weights)
    assert_same_outputs(Lf, Lu)
    del Lf, Lu, weights
    torch.cuda.empty_cache()


def test_fused_max_shapes():
    """E = 1024, k = 32, R = 1024 ranks of one expert each: 4096 group records, every tile
    partial."""
    w = I.small_workload("max", 1024, 1024, 32, 1024, 3, 128, 128, alpha=0.2, seed=13)
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    Lf = run_gpu(w, logits, x, weights, fused=True)
    if ref["err"]:
        assert int(Lf.err.item()) == ref["err"]
        return
    Lu = run_gpu(w, logits, x, weights)
    check_integer_parity(Lf, w, ref)
    assert_same_outputs(Lf, Lu)


def test_fused_graph_replay_equals_eager():
    w = I.small_workload("graph", 768, 64, 6, 8, 8, 512, 384, alpha=0.8, seed=21)
    logits, x, weights = make_inputs(w)
    W1, W3, W2 = weights
    lg, xd = logits.cuda(), x.cuda()
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F, fused=True)
    L.forward(lg, xd, W1, W3, W2)
    torch.cuda.synchronize()
    eager = L.out.clone()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        L.forward(lg, xd, W1, W3, W2)  # warm-up on the capture stream
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        L.forward(lg, xd, W1, W3, W2)
    L.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    assert torch.equal(L.out, eager)
    # new inputs through the same graph
    xd.copy_(torch.flip(xd, dims=[0]))
    g.replay()
    torch.cuda.synchronize()
    replay2 = L.out.clone()
    L.forward(lg, xd, W1, W3, W2)
    torch.cuda.synchronize()
    assert torch.equal(replay2, L.out)
    del g


def test_fused_host_pipeline_equals_unfused():
    """Host batches through HostPipeline: the fused layer frees an input slot only after the
    FFN has gathered from it; outputs equal the unfused layer's bit for bit."""
    w = I.small_workload("pipe", 512, 32, 4, 8, 4, 256, 256, alpha=1.0, seed=23)
    _, _, weights = make_inputs(w)
    W1, W3, W2 = weights
    g = torch.Generator().manual_seed(5)
    batches = []
    for _ in range(5):
        lg = torch.randn(w.T, w.E, generator=g).pin_memory()
        xb = torch.randn(w.T, w.d, generator=g).to(torch.bfloat16).pin_memory()
        batches.append((lg, xb))
    outs = {}
    for fused in (False, True):
        L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F, fused=fused)
        P = HostPipeline(L, W1, W3, W2)
        o = [torch.empty(w.T, w.d, dtype=torch.bfloat16).pin_memory() for _ in batches]
        P.run(batches, o)
        P.done().synchronize()
        torch.cuda.synchronize()
        assert int(L.err.item()) == 0
        outs[fused] = o
    for a, b in zip(outs[False], outs[True]):
        assert torch.equal(a, b)
