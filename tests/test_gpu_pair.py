"""Grouped FFN in CTA-pair mode (needs a B200).

moe_set_ffn_tile_mode(1) runs both GEMMs as 2-CTA clusters on 256-row tiles
(tcgen05.mma.cta_group::2): each CTA holds 128 rows of A and half of B, the pair shares
one 256 x N accumulator tile; a group's last block with at most 128 rows left runs as a
half tile (an M = 128 pair MMA, 64 rows per CTA; in GEMM 1 the up half of each row reaches
the gate half through shared memory).  The bar is the default tiling's: integer outputs bit-exact,
h / y / out within 1e-2 * max(1, |oracle|) (every row for small shapes, sampled tokens at
full size).  Both tilings add the same products in the same K order, so their outputs are
also compared with each other element by element.
"""
import numpy as np
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I

from harness import (check_ffn_combine_full, check_ffn_combine_sampled, check_integer_parity,
                     make_inputs, oracle_integer_path, run_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    M.lib()
    yield
    M.set_ffn_tile_mode(0)


def run_mode(w, logits, x, weights, mode):
    prev = M.set_ffn_tile_mode(mode)
    try:
        return run_gpu(w, logits, x, weights)
    finally:
        M.set_ffn_tile_mode(prev)


def assert_same_ffn(Lp, Lu):
    assert torch.equal(Lp.perm, Lu.perm), "perm"
    assert torch.equal(Lp.h, Lu.h), "h"
    assert torch.equal(Lp.y, Lu.y), "y"
    assert torch.equal(Lp.out, Lu.out), "out"


SMALL = [
    I.WORKLOADS["tiny"],
    # groups of every size class against 256-row tiles: rows % 256 in (0, 128] end in a
    # half tile (64 rows per CTA, the second CTA possibly without valid rows), (128, 256)
    # in a full tile split between the CTAs
    I.small_workload("ragged", 300, 16, 4, 4, 2, 256, 384, alpha=1.0, seed=1),
    I.small_workload("mid", 1000, 64, 6, 8, 8, 512, 256, alpha=0.6, seed=2),
    # d % 256 != 0: GEMM 2 runs N = 128, each CTA loads a 64-row half of W2
    I.small_workload("k1_d384", 96, 32, 1, 8, 2, 384, 128, alpha=1.5, seed=4),
    I.small_workload("d384_wide", 640, 16, 2, 4, 4, 384, 512, alpha=0.8, seed=6),
    I.small_workload("one_rank", 64, 16, 4, 1, 0, 128, 128, alpha=1.0, seed=5),
    I.small_workload("hot", 512, 32, 4, 8, 4, 128, 256, alpha=2.5, seed=7),
    I.small_workload("wide_E", 200, 512, 8, 16, 12, 128, 128, alpha=0.3, seed=8),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_pair_layer_parity_small(w):
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    Lp = run_mode(w, logits, x, weights, 1)
    if ref["err"]:
        assert int(Lp.err.item()) == ref["err"]
        return
    assert int(Lp.err.item()) == 0
    check_integer_parity(Lp, w, ref)
    check_ffn_combine_full(Lp, w, x, weights, ref)
    assert 1 <= M.ffn_pair_clusters() <= torch.cuda.get_device_properties(0).multi_processor_count // 2


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_pair_equals_default_tiling_small(w):
    logits, x, weights = make_inputs(w)
    Lp = run_mode(w, logits, x, weights, 1)
    Lu = run_mode(w, logits, x, weights, 0)
    assert int(Lp.err.item()) == int(Lu.err.item())
    if int(Lu.err.item()) == 0:
        assert_same_ffn(Lp, Lu)


@pytest.mark.parametrize("name", ["near_balanced", "qwen_mv15", "mixtral", "deepseek"])
def test_pair_full_size(name):
    w = I.WORKLOADS[name]
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    Lp = run_mode(w, logits, x, weights, 1)
    assert int(Lp.err.item()) == 0
    check_integer_parity(Lp, w, ref)
    rng = np.random.default_rng(19)
    tokens = sorted(rng.choice(w.T, size=6, replace=False).tolist()) + [w.T - 1]
    check_ffn_combine_sampled(Lp, w, x, weights, ref, tokens)
    Lu = run_mode(w, logits, x, weights, 0)
    assert_same_ffn(Lp, Lu)
    del Lp, Lu, weights
    torch.cuda.empty_cache()


def test_pair_max_shapes():
    """E = 1024, k = 32, R = 1024 ranks of one expert each: 4096 group records, every tile
    partial and most pair tiles with an idle second CTA."""
    w = I.small_workload("max", 1024, 1024, 32, 1024, 3, 128, 128, alpha=0.2, seed=13)
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    Lp = run_mode(w, logits, x, weights, 1)
    if ref["err"]:
        assert int(Lp.err.item()) == ref["err"]
        return
    check_integer_parity(Lp, w, ref)
    Lu = run_mode(w, logits, x, weights, 0)
    assert_same_ffn(Lp, Lu)


def test_pair_error_word_stops_the_ffn():
    """A plan error (more replicas than slots) set before the FFN: both CTAs of every pair
    skip all tiles, h and y keep their contents."""
    w = I.small_workload("noslots", 64, 16, 4, 4, 0, 128, 128, alpha=200.0, seed=10)
    logits, x, weights = make_inputs(w)
    prev = M.set_ffn_tile_mode(1)
    try:
        L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
        L.h.fill_(5.0)
        L.y.fill_(6.0)
        L.forward(logits.cuda(), x.cuda(), *weights)
        torch.cuda.synchronize()
    finally:
        M.set_ffn_tile_mode(prev)
    assert int(L.err.item()) == M.DERR_SLOTS
    assert bool((L.h == 5.0).all()) and bool((L.y == 6.0).all())


def test_pair_graph_replay_equals_eager():
    w = I.small_workload("graph", 768, 64, 6, 8, 8, 512, 384, alpha=0.8, seed=21)
    logits, x, weights = make_inputs(w)
    W1, W3, W2 = weights
    lg, xd = logits.cuda(), x.cuda()
    prev = M.set_ffn_tile_mode(1)
    try:
        L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
        L.forward(lg, xd, W1, W3, W2)
        torch.cuda.synchronize()
        eager = L.out.clone()
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            L.forward(lg, xd, W1, W3, W2)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            L.forward(lg, xd, W1, W3, W2)
        L.out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert int(L.err.item()) == 0
        assert torch.equal(L.out, eager)
        del g
    finally:
        M.set_ffn_tile_mode(prev)


def test_tile_mode_argument_checked():
    prev = M.set_ffn_tile_mode(0)
    with pytest.raises(M.MoEError):
        M.set_ffn_tile_mode(2)
    assert M.set_ffn_tile_mode(prev) == 0
