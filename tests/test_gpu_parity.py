"""CUDA path vs the CPU oracle, call by call, through the C ABI (needs a B200).

Integer outputs (top-k ids, counts, loads, maxvio, the plan, perm/src, recv rows, pool
slots) must be bit-exact; gates within 1e-6; h, y and out within 1e-2*max(1,|oracle|).
Small shapes compare every element; the full-size workloads compare every integer output
and a sample of tokens for the floating-point ones.
"""
import json
import os

import numpy as np
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I
from oracle import moe_oracle as O

from harness import (check_ffn_combine_full, check_ffn_combine_sampled, check_ffn_edge_rows,
                     check_integer_parity, check_rows_and_pool, edge_rows, make_inputs,
                     oracle_integer_path, run_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    M.lib()


SMALL = [
    I.WORKLOADS["tiny"],
    I.small_workload("ragged", 300, 16, 4, 4, 2, 256, 384, alpha=1.0, seed=1),
    I.small_workload("mid", 1000, 64, 6, 8, 8, 512, 256, alpha=0.6, seed=2),
    I.small_workload("k_eq_E", 64, 8, 8, 4, 2, 128, 128, alpha=0.0, seed=3),
    I.small_workload("k1_d384", 96, 32, 1, 8, 2, 384, 128, alpha=1.5, seed=4),
    I.small_workload("one_rank", 64, 16, 4, 1, 0, 128, 128, alpha=1.0, seed=5),
    I.small_workload("rank_per_expert", 256, 8, 2, 8, 3, 256, 256, alpha=0.5, seed=6),
    I.small_workload("hot", 512, 32, 4, 8, 4, 128, 256, alpha=2.5, seed=7),
    I.small_workload("wide_E", 200, 512, 8, 16, 12, 128, 128, alpha=0.3, seed=8),
    I.small_workload("wide_E_few_slots", 200, 512, 8, 16, 4, 128, 128, alpha=0.3, seed=8),
    # one token: C = 1 row per rank, single-row groups and tiles
    I.small_workload("single_token", 1, 8, 2, 2, 2, 128, 128, alpha=1.0, seed=15),
    # one token per expert slot: T*k/R = 1 with every rank's row a replica or a home row
    I.small_workload("one_row_per_rank", 4, 16, 4, 16, 1, 256, 128, alpha=0.0, seed=16),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_layer_parity_small(w):
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    L = run_gpu(w, logits, x, weights)
    if ref["err"]:
        assert int(L.err.item()) == ref["err"]
        return
    check_integer_parity(L, w, ref)
    check_rows_and_pool(L, w, x, weights, ref)
    check_ffn_combine_full(L, w, x, weights, ref)


FULL = ["near_balanced", "qwen_mv0.2", "qwen_mv1", "qwen_mv5", "qwen_mv15", "mixtral", "deepseek"]


@pytest.mark.parametrize("name", FULL)
def test_layer_parity_full_size(name):
    w = I.WORKLOADS[name]
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    assert ref["err"] == 0
    L = run_gpu(w, logits, x, weights)
    check_integer_parity(L, w, ref)
    check_rows_and_pool(L, w, x, weights, ref)
    # every rank holds exactly C rows: the plan's groups tile [u*C, (u+1)*C)
    rng = np.random.default_rng(11)
    tokens = sorted(rng.choice(w.T, size=8, replace=False).tolist()) + [w.T - 1]
    check_ffn_combine_sampled(L, w, x, weights, ref, tokens)
    # h and y at the rows where tiling breaks: the last partial tile of the largest group,
    # a 128-row tile boundary, a replica group, the last group of the last rank
    sets = check_ffn_edge_rows(L, w, x, weights, ref)
    assert len(sets) == 4, sorted(sets)
    del L, weights
    torch.cuda.empty_cache()


def test_histogram_fixture_mappings_on_gpu():
    """The pages' 16-token trace through moe_histogram_maxvio under both mappings."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hotspot_fixture.json")))
    idx = torch.tensor([[int(p[0]), int(p[1])] for p in g["pairs"]], dtype=torch.int32, device="cuda")
    for mapping, loads_exp, bal in ((g["initial_mapping"], g["initial_rank_demand"], 8 / 15),
                                    (g["proposed_mapping"], g["proposed_rank_demand"], 0.8)):
        m = torch.zeros(8, dtype=torch.int32)
        for r, es in enumerate(mapping):
            m[es] = r
        counts = torch.empty(8, dtype=torch.int32, device="cuda")
        loads = torch.empty(4, dtype=torch.int32, device="cuda")
        mv = torch.empty(1, dtype=torch.float64, device="cuda")
        b = torch.empty(1, dtype=torch.float64, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        M.moe_histogram_maxvio(idx, 8, 4, counts, loads, mv, b, err, expert_to_rank=m.cuda())
        torch.cuda.synchronize()
        assert err.item() == 0
        assert counts.tolist() == g["expert_demand"]
        assert loads.tolist() == loads_exp
        assert b.item() == bal
        assert mv.item() == max(loads_exp) / 8 - 1


def _hist(idx, E, R):
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    loads = torch.empty(R, dtype=torch.int32, device="cuda")
    mv = torch.empty(1, dtype=torch.float64, device="cuda")
    b = torch.empty(1, dtype=torch.float64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_histogram_maxvio(idx, E, R, counts, loads, mv, b, err)
    torch.cuda.synchronize()
    return int(err.item())


def test_trace_validation_errors():
    good = torch.tensor([[0, 1], [2, 3], [4, 5]], dtype=torch.int32, device="cuda")
    assert _hist(good, 8, 4) == 0
    bad = good.clone()
    bad[1, 1] = 8
    assert _hist(bad, 8, 4) == M.DERR_ID_RANGE
    bad[1, 1] = -3
    assert _hist(bad, 8, 4) == M.DERR_ID_RANGE
    dup = good.clone()
    dup[2, 1] = 4
    assert _hist(dup, 8, 4) == M.DERR_DUPLICATE


def _hist_full(idx, E, R, expert_to_rank=None):
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    loads = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    mv = torch.full((1,), -7.0, dtype=torch.float64, device="cuda")
    b = torch.full((1,), -7.0, dtype=torch.float64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_histogram_maxvio(idx, E, R, counts, loads, mv, b, err, expert_to_rank=expert_to_rank)
    torch.cuda.synchronize()
    return dict(err=int(err.item()), counts=counts.cpu().numpy(), loads=loads.cpu().numpy(),
                maxvio=float(mv.item()), balancedness=float(b.item()))


def _same_as_oracle(got, ref):
    assert got["err"] == ref["err"]
    assert np.array_equal(got["counts"], ref["counts"])
    assert np.array_equal(got["loads"], ref["loads"])
    assert got["maxvio"] == ref["maxvio"] and got["balancedness"] == ref["balancedness"]


def test_histogram_mapping_missing_an_expert():
    """"If any expert is missing from a mapping, stop": a map entry outside [0, R) sets
    MOE_DERR_ID_RANGE, and the GPU's counts, loads, maxvio and balancedness equal the
    oracle's (the unmapped expert's demand goes to no rank)."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hotspot_fixture.json")))
    idx_h = np.array([[int(p[0]), int(p[1])] for p in g["pairs"]], dtype=np.int32)
    idx = torch.from_numpy(idx_h).cuda()
    base = np.zeros(8, dtype=np.int32)
    for r, es in enumerate(g["initial_mapping"]):
        base[es] = r
    for e, r in ((7, -1), (0, 4), (3, -4), (5, 1 << 20)):
        m = base.copy()
        m[e] = r
        ref = O.expert_histogram(idx_h, 8, 4, m)
        assert ref["err"] == O.ERR_ID_RANGE
        _same_as_oracle(_hist_full(idx, 8, 4, torch.from_numpy(m).cuda()), ref)


def test_histogram_errors_found_in_different_blocks():
    """A trace spread over every block of the histogram grid, with an unknown id in the
    first token and a repeated expert in the last: both error bits, and the counts of all
    in-range ids, whatever order the blocks run in (five calls, identical results)."""
    T, k, E, R = 65536, 8, 256, 32
    rng = np.random.default_rng(21)
    idx_h = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    idx_h[0, 3] = E + 5
    idx_h[T - 1, 6] = idx_h[T - 1, 2]
    ref = O.expert_histogram(idx_h, E, R)
    assert ref["err"] == O.ERR_ID_RANGE | O.ERR_DUPLICATE
    idx = torch.from_numpy(idx_h).cuda()
    for _ in range(5):
        _same_as_oracle(_hist_full(idx, E, R), ref)


def test_nonfinite_logit_stops_the_layer():
    w = I.small_workload("nan", 64, 8, 2, 4, 2, 128, 128, alpha=1.0, seed=9)
    logits, x, weights = make_inputs(w)
    for bad in (float("nan"), float("inf"), float("-inf")):
        lg = logits.clone()
        lg[17, 3] = bad
        L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
        L.out.fill_(7.0)
        L.forward(lg.cuda(), x.cuda(), *weights)
        torch.cuda.synchronize()
        assert int(L.err.item()) == M.DERR_NONFINITE
        assert bool((L.out == 7.0).all()), "calls after an error must not run"


def test_slot_overflow_sets_error_and_stops():
    # all tokens on experts 0..3 (rank 0) and no prefetch slots: replicas are needed
    w = I.small_workload("noslots", 64, 16, 4, 4, 0, 128, 128, alpha=200.0, seed=10)
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    assert ref["err"] == O.ERR_SLOTS
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    L.recv.fill_(3.0)
    L.forward(logits.cuda(), x.cuda(), *weights)
    torch.cuda.synchronize()
    assert int(L.err.item()) == M.DERR_SLOTS
    assert bool((L.recv == 3.0).all())


def test_empty_batch():
    w = I.small_workload("empty", 0, 8, 2, 4, 2, 128, 128)
    W = I.make_weights(w, device="cuda")
    L = M.MoELayer(0, 8, 2, 4, 2, 128, 128)
    L.forward(torch.empty(0, 8, device="cuda"), torch.empty(0, 128, dtype=torch.bfloat16, device="cuda"), *W)
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    assert L.maxvio.item() == 0.0 and L.balancedness.item() == 1.0
    assert L.counts.tolist() == [0] * 8 and L.loads.tolist() == [0] * 4


@pytest.mark.parametrize("E,k", [(64, 6), (256, 8), (100, 5)])
def test_topk_ties_and_signed_zero(E, k):
    T = 512
    g = torch.Generator().manual_seed(12)
    vals = torch.tensor([-1.0, -0.0, 0.0, 0.5, 2.0])
    logits = vals[torch.randint(0, 5, (T, E), generator=g)].contiguous()
    idx_ref, gate_ref, err = O.topk_route(logits.numpy(), k)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    e = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_topk(logits.cuda(), k, idx, gate, e)
    torch.cuda.synchronize()
    assert e.item() == 0
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.abs(gate.cpu().double().numpy() - gate_ref).max() <= 1e-6


@pytest.mark.parametrize("E", [1, 3, 33, 100, 257, 700, 1024])
def test_topk_expert_counts(E):
    T = 333
    k = min(E, 8)
    logits = torch.randn(T, E, generator=torch.Generator().manual_seed(E))
    idx_ref, gate_ref, _ = O.topk_route(logits.numpy(), k)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    e = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_topk(logits.cuda(), k, idx, gate, e)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.abs(gate.cpu().double().numpy() - gate_ref).max() <= 1e-6


@pytest.mark.parametrize("E,k", [(256, 8), (64, 6), (128, 8), (8, 2)])
def test_topk_many_tokens_staged_rows(E, k):
    """Many tokens through the stand-alone top-k: the DeepSeek workload's logits, then
    T = 20001 random rows (the last block of 8 warps holds one token) with every fifth row
    made of ties (the exact path)."""
    if E == 256:
        w = I.WORKLOADS["deepseek"]
        logits = I.make_logits(w)
    else:
        g = torch.Generator().manual_seed(E + k)
        logits = torch.randn(20001, E, generator=g)
        vals = torch.tensor([-1.0, -0.0, 0.0, 0.5, 2.0])
        tie = vals[torch.randint(0, 5, (4001, E), generator=g)]
        logits[::5] = tie
    T = logits.shape[0]
    idx_ref, gate_ref, err = O.topk_route(logits.numpy(), k)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    e = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_topk(logits.cuda(), k, idx, gate, e)
    torch.cuda.synchronize()
    assert e.item() == 0
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.abs(gate.cpu().double().numpy() - gate_ref).max() <= 1e-6


def test_topk_biased_many_tokens():
    """Bias-only selection over 113741 tokens (14218 blocks, a ragged last block) with
    ties on every seventh row: ids bit-exact against the oracle, gates within 1e-6."""
    T, E, k = 113741, 128, 6
    g = torch.Generator().manual_seed(61)
    logits = torch.randn(T, E, generator=g)
    vals = torch.tensor([-1.0, -0.0, 0.0, 0.5, 2.0])
    logits[::7] = vals[torch.randint(0, 5, logits[::7].shape, generator=g)]
    bias = torch.randn(E, generator=g) * 0.5
    idx_ref, gate_ref, err = O.topk_route_biased(logits.numpy(), bias.numpy(), k)
    assert err == 0
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    e = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_topk_biased(logits.cuda(), bias.cuda(), k, idx, gate, e)
    torch.cuda.synchronize()
    assert e.item() == 0
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.abs(gate.cpu().double().numpy() - gate_ref).max() <= 1e-6


def test_topk_resets_a_stale_error_word_before_the_next_call():
    """moe_topk starts while its error-word reset is still finishing (a programmatic
    dependent launch): a stale non-zero word must read 0 after a clean call, so that the
    histogram launched next on the stream runs, and exactly NONFINITE after a call with one
    non-finite logit in the last token; both inside one CUDA graph replayed twice."""
    T, E, k, R = 4096, 256, 8, 32
    g = torch.Generator().manual_seed(77)
    clean = torch.randn(T, E, generator=g).cuda()
    bad = clean.clone()
    bad[T - 1, 5] = float("nan")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    err = torch.empty(1, dtype=torch.int32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    loads = torch.empty(R, dtype=torch.int32, device="cuda")
    mv = torch.empty(1, dtype=torch.float64, device="cuda")
    bal = torch.empty(1, dtype=torch.float64, device="cuda")
    err_after = torch.empty(2, dtype=torch.int32, device="cuda")
    counts_after = torch.empty(E, dtype=torch.int32, device="cuda")
    idx_ref, _, _ = O.topk_route(clean.cpu().numpy(), k)
    counts_ref = np.bincount(idx_ref.reshape(-1), minlength=E)

    def step():
        err.fill_(0x7F)  # stale bits from an earlier step
        M.moe_topk(clean, k, idx, gate, err)
        M.moe_histogram_maxvio(idx, E, R, counts, loads, mv, bal, err)
        err_after[0:1].copy_(err)
        counts_after.copy_(counts)
        err.fill_(0x7F)
        M.moe_topk(bad, k, idx, gate, err)
        err_after[1:2].copy_(err)

    step()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        graph.capture_begin()
        step()
        graph.capture_end()
    torch.cuda.synchronize()
    for _ in range(2):
        err_after.fill_(-1)
        counts_after.fill_(-1)
        graph.replay()
        torch.cuda.synchronize()
        assert err_after.tolist() == [0, M.DERR_NONFINITE]
        assert np.array_equal(counts_after.cpu().numpy(), counts_ref)
    del graph


def test_bounded_wait_gives_up_and_context_survives():
    """The FFN's bounded mbarrier wait, on a barrier nothing arrives at, returns with the
    timeout bit; the next layer on the same context still matches the oracle."""
    import time
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    M.moe_selftest_bounded_wait(err, limit_us=20000)
    torch.cuda.synchronize()
    assert err.item() == M.DERR_TIMEOUT
    assert time.time() - t0 < 5.0
    w = I.WORKLOADS["tiny"]
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    L = run_gpu(w, logits, x, weights)
    check_integer_parity(L, w, ref)
    check_ffn_combine_full(L, w, x, weights, ref)


def test_many_tile_dispatch():
    """98304 tokens = 384 placement tiles of 256: the rank pass looks back over a dozen
    windows of 32 predecessor tiles; perm, src and the received rows stay bit-exact."""
    w = I.small_workload("tiles", 98304, 64, 4, 8, 8, 128, 128, alpha=0.5, seed=14)
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    assert ref["err"] == 0
    L = run_gpu(w, logits, x, weights)
    check_integer_parity(L, w, ref)
    check_rows_and_pool(L, w, x, weights, ref)


def test_max_shapes():
    """Limits of the boundary: E = 1024 experts, k = 32, R = 1024 ranks (B = 1), S = 3 slots
    (R*(B+S) = 4096 group records), through the whole layer."""
    w = I.small_workload("max", 1024, 1024, 32, 1024, 3, 128, 128, alpha=0.2, seed=13)
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    L = run_gpu(w, logits, x, weights)
    if ref["err"]:
        assert int(L.err.item()) == ref["err"]
        return
    check_integer_parity(L, w, ref)
    check_rows_and_pool(L, w, x, weights, ref)
    check_ffn_combine_full(L, w, x, weights, ref)
