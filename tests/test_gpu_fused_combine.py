"""Combine folded into GEMM 2's epilogue (moe_grouped_ffn_combine) against the CPU oracle
(needs a B200).

out[t] = sum_j gate[t,j] * y[perm[t,j]] accumulated from the tensor-core accumulator in
fp32 with atomics, in no fixed order: every token of small shapes and sampled tokens of
the full-size workloads within 1e-2 * max(1, |oracle|), and the whole output within twice
that of the unfused path's (each is within the bound of the fp64 result).
"""
import numpy as np
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I
from oracle import moe_oracle as O

from harness import (assert_close_scaled, expert_weights64, make_inputs, oracle_integer_path,
                     to64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    M.lib()


def _run(w, logits, x, weights, fused_combine):
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F, fused_combine=fused_combine)
    L.forward(logits.cuda(), x.cuda(), *weights)
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    return L


def _oracle_out(w, L, weights, ref, tokens):
    rows = sorted({int(r) for t in tokens for r in ref["perm"][t]})
    recv = to64(L.recv[torch.tensor(rows, device="cuda")])
    row_e = {}
    for gl in ref["plan"]["groups"]:
        for (r0, n, e, _) in gl:
            for r in rows:
                if r0 <= r < r0 + n:
                    row_e[r] = e
    y = {}
    by_e = {}
    for i, r in enumerate(rows):
        by_e.setdefault(row_e[r], []).append(i)
    for e, ii in by_e.items():
        w1, w3, w2 = expert_weights64(weights, e)
        ys = O.expert_ffn(recv[ii], w1, w3, w2)
        for i, yr in zip(ii, ys):
            y[rows[i]] = yr
    return O.combine(y, ref["perm"], ref["gate"], tokens=tokens)


SMALL = [
    I.WORKLOADS["tiny"],
    I.small_workload("ragged", 300, 16, 4, 4, 2, 256, 384, alpha=1.0, seed=1),
    I.small_workload("mid", 1000, 64, 6, 8, 8, 512, 256, alpha=0.6, seed=2),
    I.small_workload("k1_d384", 96, 32, 1, 8, 2, 384, 128, alpha=1.5, seed=4),
    I.small_workload("hot", 512, 32, 4, 8, 4, 128, 256, alpha=2.5, seed=7),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_fused_combine_small(w):
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    assert ref["err"] == 0
    L = _run(w, logits, x, weights, True)
    assert L.y is None
    tokens = list(range(w.T))
    out_ref = _oracle_out(w, L, weights, ref, tokens)
    assert_close_scaled(to64(L.out), np.stack([out_ref[t] for t in tokens]), "out (fused combine)")


@pytest.mark.parametrize("name", ["near_balanced", "qwen_mv1", "deepseek"])
def test_fused_combine_full_size(name):
    w = I.WORKLOADS[name]
    logits, x, weights = make_inputs(w)
    ref = oracle_integer_path(w, logits)
    Lf = _run(w, logits, x, weights, True)
    assert np.array_equal(Lf.perm.cpu().numpy(), ref["perm"])
    rng = np.random.default_rng(23)
    tokens = sorted(rng.choice(w.T, size=8, replace=False).tolist()) + [w.T - 1]
    out_ref = _oracle_out(w, Lf, weights, ref, tokens)
    got = to64(Lf.out[torch.tensor(tokens, device="cuda")])
    assert_close_scaled(got, np.stack([out_ref[t] for t in tokens]), "out (fused combine, sampled)")
    out_f = Lf.out.clone()
    del Lf
    Lu = _run(w, logits, x, weights, False)
    a, b = out_f.double(), Lu.out.double()
    bad = ((a - b).abs() > 2e-2 * b.abs().clamp(min=1.0)).sum().item()
    assert bad == 0, f"{bad} elements differ from the unfused combine by more than twice the bound"
    del Lu, weights
    torch.cuda.empty_cache()


def test_fused_combine_graph_replay():
    w = I.small_workload("mid", 1000, 64, 6, 8, 8, 512, 256, alpha=0.6, seed=2)
    logits, x, weights = make_inputs(w)
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F, fused_combine=True)
    lg, xd = logits.cuda(), x.cuda()
    L.forward(lg, xd, *weights)
    torch.cuda.synchronize()
    eager = L.out.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g.capture_begin()
        L.forward(lg, xd, *weights)
        g.capture_end()
    torch.cuda.synchronize()
    L.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    a, b = L.out.double(), eager.double()
    assert ((a - b).abs() <= 1e-2 * b.abs().clamp(min=1.0)).all()


def test_fused_combine_host_pipeline():
    """The host-to-host pipeline with a fused-combine layer: each batch's output equals the
    same layer's forward on that batch (within the bound: atomic order)."""
    from load_balanced_dispatch_warp_b200.pipeline import HostPipeline
    w = I.small_workload("mid", 1000, 64, 6, 8, 8, 512, 256, alpha=0.6, seed=2)
    logits, x, weights = make_inputs(w)
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F, fused_combine=True)
    pipe = HostPipeline(L, *weights)
    outs = [torch.empty(w.T, w.d, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    pipe.run([(logits.pin_memory(), x.pin_memory())] * 3, outs)
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    ref = L.forward(logits.cuda(), x.cuda(), *weights).double().cpu()
    torch.cuda.synchronize()
    for o in outs:
        assert ((o.double() - ref).abs() <= 1e-2 * ref.abs().clamp(min=1.0)).all()
