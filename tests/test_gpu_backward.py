"""Backward pass on the GPU vs the oracle's fp64 chain rule (needs a B200).

Outputs: dy and dgate (combine backward), the dX rows and the expert weight gradients dW1,
dW3, dW2 (grouped FFN backward, replica gradients reduced to the home experts), dx
(dispatch backward) and dlogits (gate backward).  Each kernel is checked against the
oracle given the GPU's own inputs, then the whole backward against the fp64 chain rule.

Tolerance, derived from the arithmetic: every GEMM output is a sum of products whose one
operand the GPU rounds to bf16 before the fp32 accumulation (dY, dG, dU, and W2 and h on
their way into the transposed operands).  bf16 carries 8 significant bits, so one rounding
moves a value by at most 2^-8 of itself (h is rounded twice: fp16 in the forward, then
bf16), and |gpu - oracle| <= (2^-8 + 2^-11) * sum |terms| up to fp32 accumulation.  Each
kernel is allowed 2^-7 * sum |terms| + 1e-5, with sum |terms| from the oracle's values
(|dG|^T |X| for dW1, and so on); the whole backward against the fp64 chain rule twice
that.  Where a sum does not cancel this is about 1e-2 relative or tighter; where it
cancels, the bound follows the magnitude of the terms, as the rounding does.  dgate and
dlogits (dot products of dout with the bf16 forward output y) use the same form.
"""
import numpy as np
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I
from oracle import moe_oracle as O

from harness import assert_close_scaled, make_inputs, run_gpu, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    M.lib()


def dout_for(w, seed=31):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(w.T, w.d, generator=g).to(torch.bfloat16)


SMALL = [
    I.WORKLOADS["tiny"],
    I.small_workload("ragged", 300, 16, 4, 4, 2, 256, 384, alpha=1.0, seed=1),
    I.small_workload("mid", 1000, 64, 6, 8, 8, 512, 256, alpha=0.6, seed=2),
    I.small_workload("k1_d384", 96, 32, 1, 8, 2, 384, 128, alpha=1.5, seed=4),
    I.small_workload("one_rank", 64, 16, 4, 1, 0, 128, 128, alpha=1.0, seed=5),
    I.small_workload("hot", 512, 32, 4, 8, 4, 128, 256, alpha=2.5, seed=7),
    # 512 experts for 200 tokens: many experts receive no rows (zero gradients)
    I.small_workload("wide_E", 200, 512, 8, 16, 12, 128, 128, alpha=0.3, seed=8),
]


TOL = 2.0 ** -7


def magnitudes(w, X, dy, plan, W64, g, propagate=False):
    """sum |terms| of every GEMM output of the FFN backward (the oracle's values).  With
    propagate, the rounding of dy is carried through dH = dY W2, which can cancel: the
    magnitude of dG is then |u silu'(g)| (|dY| |W2|) instead of |dG| (and alike for dU)."""
    W1, W3, W2 = W64
    dX = np.zeros_like(g["dX"] if "dX" in g else g["dX_rows"])
    dW1 = np.zeros_like(g["dW1"])
    dW3 = np.zeros_like(g["dW3"])
    dW2 = np.zeros_like(g["dW2"])
    for u_groups in plan["groups"]:
        for (r0, n, e, ref) in u_groups:
            sl = slice(r0, r0 + n)
            Xg = np.abs(X[sl])
            gg = X[sl] @ W1[e].T
            uu = X[sl] @ W3[e].T
            h = np.abs(O.silu(gg) * uu)
            if propagate:
                dhm = np.abs(dy[sl]) @ np.abs(W2[e])
                dg = dhm * np.abs(uu * O.silu_grad(gg))
                du = dhm * np.abs(O.silu(gg))
            else:
                dg = np.abs(g["dg"][sl])
                du = np.abs(g["du"][sl])
            dX[sl] = dg @ np.abs(W1[e]) + du @ np.abs(W3[e])
            dW1[e] += dg.T @ Xg
            dW3[e] += du.T @ Xg
            dW2[e] += np.abs(dy[sl]).T @ h
    return dict(dX=dX, dW1=dW1, dW3=dW3, dW2=dW2)


def assert_within(gpu, ref, bound, what):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bad = np.abs(gpu - ref) > bound
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside; first at {i}: "
                             f"gpu {gpu[i]} oracle {ref[i]} bound {np.broadcast_to(bound, gpu.shape)[i]}")


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_backward_parity_small(w):
    logits, x, weights = make_inputs(w)
    L = run_gpu(w, logits, x, weights)
    assert int(L.err.item()) == 0
    dout = dout_for(w)
    W1, W3, W2 = weights
    b = L.backward(dout.cuda(), W1, W3, W2)
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    W64 = [to64(t) for t in weights]
    fwd = O.layer(logits.numpy(), to64(x), W64[0], W64[1], W64[2], w.k, w.R, w.S)
    assert fwd["err"] == 0
    if w.name == "hot":
        assert sum(1 for e in fwd["plan"]["replica_expert"] if e >= 0) >= 1
    ref = O.layer_backward(fwd, to64(dout), W64[0], W64[1], W64[2], w.E)
    d64 = to64(dout)
    perm = fwd["perm"]
    # each kernel against the oracle given the GPU's own inputs
    y_gpu = to64(L.y)
    dy_iso, dgate_iso = O.combine_backward(d64, y_gpu, perm, to64(L.gate))
    assert_close_scaled(to64(b["dy"]), dy_iso, "dy")
    terms = np.stack([np.abs(d64[t]) @ np.abs(y_gpu[perm[t]].T) for t in range(w.T)]) if w.T else 0
    assert_within(to64(b["dgate"]), dgate_iso, 1e-4 * np.maximum(1.0, terms), "dgate (kernel)")
    g_iso = O.grouped_ffn_backward(to64(x)[fwd["src"]], to64(b["dy"]), fwd["plan"], w.E, W64[0],
                                   W64[1], W64[2], fwd["pool"])
    mag = magnitudes(w, to64(x)[fwd["src"]], to64(b["dy"]), fwd["plan"], W64, g_iso)
    assert_within(to64(b["dx_rows"]), g_iso["dX"], TOL * mag["dX"] + 1e-5, "dX rows")
    assert_within(to64(b["dW1"]), g_iso["dW1"], TOL * mag["dW1"] + 1e-5, "dW1")
    assert_within(to64(b["dW3"]), g_iso["dW3"], TOL * mag["dW3"] + 1e-5, "dW3")
    assert_within(to64(b["dW2"]), g_iso["dW2"], TOL * mag["dW2"] + 1e-5, "dW2")
    dx_iso = O.dispatch_backward(to64(b["dx_rows"]), perm)
    assert_within(to64(b["dx"]), dx_iso, TOL * O.dispatch_backward(np.abs(to64(b["dx_rows"])), perm) + 1e-5,
                  "dx (kernel)")
    dl_iso = O.topk_backward(to64(L.gate), to64(b["dgate"]), fwd["idx"], w.E)
    assert_within(to64(b["dlogits"]), dl_iso, 1e-5 * np.maximum(1.0, np.abs(dl_iso)), "dlogits (kernel)")
    # end to end against the fp64 chain rule (the oracle's own dy and y), twice the bound
    mag_ref = magnitudes(w, to64(x)[fwd["src"]], ref["dy"], fwd["plan"], W64, ref, propagate=True)
    for key in ("dW1", "dW3", "dW2"):
        assert_within(to64(b[key]), ref[key], 2 * TOL * mag_ref[key] + 1e-5, f"{key} (end to end)")
    assert_within(to64(b["dx"]), ref["dx"],
                  2 * TOL * O.dispatch_backward(mag_ref["dX"], perm) + 1e-5, "dx (end to end)")
    assert_within(to64(b["dgate"]), ref["dgate"], 2 * TOL * terms + 1e-5, "dgate (end to end)")
    scale = np.zeros((w.T, w.E))
    for t in range(w.T):
        s_t = float(to64(L.gate)[t] @ terms[t])
        for j in range(w.k):
            scale[t, fwd["idx"][t, j]] = to64(L.gate)[t, j] * (terms[t, j] + s_t)
    assert_within(to64(b["dlogits"]), ref["dlogits"], 2 * TOL * scale + 1e-5, "dlogits (end to end)")
    if w.name == "wide_E":
        counts = np.bincount(np.asarray(fwd["idx"]).reshape(-1), minlength=w.E)
        empty = np.nonzero(counts == 0)[0]
        assert len(empty) > 0
        assert not b["dW1"][torch.from_numpy(empty).cuda()].any()


def test_backward_twice_reuses_buffers():
    """A second backward on new dout overwrites every output (no stale accumulation)."""
    w = I.small_workload("twice", 256, 16, 4, 4, 2, 128, 128, alpha=1.0, seed=9)
    logits, x, weights = make_inputs(w)
    L = run_gpu(w, logits, x, weights)
    W1, W3, W2 = weights
    d1 = dout_for(w, 1).cuda()
    d2 = dout_for(w, 2).cuda()
    first = {k: v.clone() for k, v in L.backward(d1, W1, W3, W2).items() if k != "workspace"}
    L.backward(d2, W1, W3, W2)
    again = L.backward(d1, W1, W3, W2)
    torch.cuda.synchronize()
    for key, v in first.items():
        assert torch.equal(v, again[key]), key


@pytest.mark.parametrize("name", ["near_balanced", "deepseek"])
def test_ffn_backward_full_size_busiest_experts(name):
    w = I.WORKLOADS[name]
    logits, x, weights = make_inputs(w)
    L = run_gpu(w, logits, x, weights)
    assert int(L.err.item()) == 0
    W1, W3, W2 = weights
    b = L.backward(dout_for(w).cuda(), W1, W3, W2)
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    groups = L.plan_field("groups").view(-1, 4).cpu().numpy()
    groups = groups[groups[:, 1] > 0]
    rows_of = {}
    for r0, n, e, ref in groups:
        rows_of.setdefault(int(e), []).append((int(r0), int(n), int(ref)))
    # the two experts with the most groups (replicated) and the most rows
    by_groups = sorted(rows_of, key=lambda e: (-len(rows_of[e]), -sum(n for _, n, _ in rows_of[e])))
    picked = by_groups[:2] if name == "near_balanced" else by_groups[:1]
    assert any(len(rows_of[e]) > 1 for e in picked), "a replicated expert must be checked"
    recv = L.recv
    dy = b["dy"]
    for e in picked:
        rows = np.concatenate([np.arange(r0, r0 + n) for r0, n, _ in rows_of[e]])
        ridx = torch.from_numpy(rows).cuda()
        X = to64(recv[ridx])
        DY = to64(dy[ridx])
        w1, w3, w2 = to64(W1[e]), to64(W3[e]), to64(W2[e])
        r = O.expert_ffn_backward(X, w1, w3, w2, DY)
        aX, adg, adu = np.abs(X), np.abs(r["dg"]), np.abs(r["du"])
        assert_within(to64(b["dW1"][e]), r["dw1"], TOL * (adg.T @ aX) + 1e-5, f"dW1[{e}]")
        assert_within(to64(b["dW3"][e]), r["dw3"], TOL * (adu.T @ aX) + 1e-5, f"dW3[{e}]")
        assert_within(to64(b["dW2"][e]), r["dw2"], TOL * (np.abs(DY).T @ np.abs(r["h"])) + 1e-5,
                      f"dW2[{e}]")
        sample = np.arange(0, len(rows), max(1, len(rows) // 64))
        mag_dx = adg[sample] @ np.abs(w1) + adu[sample] @ np.abs(w3)
        assert_within(to64(b["dx_rows"][ridx[torch.from_numpy(sample).cuda()]]), r["dX"][sample],
                      TOL * mag_dx + 1e-5, f"dX rows of expert {e}")
    del L, b, weights
    torch.cuda.empty_cache()
