"""Fixed-capacity (dropping) mode on the GPU against the CPU oracle (needs a B200).

"MoE Load Balancing: Find Expert Hotspots", section "Make expert capacity, overflow, and
padding explicit": cap = ceil(A / E * cf) rows per expert, each expert keeping its first
cap assignments in token order.  perm (with -1 for dropped assignments), src (with -1 for
padding rows) and the recv rows must be bit-exact; h, y and out within
1e-2 * max(1, |oracle|); the ledger bit-exact.  The pages' fixture, then the five workload
shapes at capacity factors 1, 1.25 and 2.
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

from harness import assert_close_scaled, make_inputs, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    M.lib()


def _expert_rows_ref(recv64, weights, E, cap, rows):
    """h and y of the given rows of the fixed-capacity buffer (row r belongs to expert
    r // cap), fp64 from the bf16/fp16 inputs."""
    W1, W3, W2 = weights
    by_e = {}
    for r in rows:
        by_e.setdefault(r // cap, []).append(r)
    h, y = {}, {}
    for e, rs in by_e.items():
        w1, w3, w2 = to64(W1[e]), to64(W3[e]), to64(W2[e])
        X = recv64[rs]
        hh = O.silu(X @ w1.T) * (X @ w3.T)
        yy = O.expert_ffn(X, w1, w3, w2)
        for i, r in enumerate(rs):
            h[r], y[r] = hh[i], yy[i]
    return h, y


def _check_rows(layer, weights, E, cap, rows, what):
    rows = sorted(set(rows))
    rt = torch.tensor(rows, device="cuda")
    recv64 = _RowView({r: v for r, v in zip(rows, to64(layer.recv[rt]))})
    h_ref, y_ref = _expert_rows_ref(recv64, weights, E, cap, rows)
    assert_close_scaled(to64(layer.h[rt]), np.stack([h_ref[r] for r in rows]), f"h, {what}")
    assert_close_scaled(to64(layer.y[rt]), np.stack([y_ref[r] for r in rows]), f"y, {what}")


class _RowView:
    """recv rows by global row index (only the rows fetched)."""

    def __init__(self, rows):
        self.rows = rows

    def __getitem__(self, rs):
        return np.stack([self.rows[r] for r in rs])


def test_fixture_fixed_capacity_on_gpu():
    """The pages' 16-token trace at cap 5: the dropped assignments (tokens 5, 6, 7, 8 of
    expert 0, token 12 of expert 1), the processed / overflow / padding ledgers, the rows of
    every expert's block, and the whole layer after them."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hotspot_fixture.json")))
    idx_h = np.array([[int(p[0]), int(p[1])] for p in g["pairs"]], dtype=np.int32)
    T, k, E, d, F = 16, 2, 8, 128, 256
    cap = M.capacity_rows(T, k, E, 5, 4)
    assert cap == 5
    gen = torch.Generator().manual_seed(3)
    x = torch.randn(T, d, generator=gen).to(torch.bfloat16)
    W1 = (torch.randn(E, F, d, generator=gen) / d ** 0.5).to(torch.bfloat16).cuda()
    W3 = (torch.randn(E, F, d, generator=gen) / d ** 0.5).to(torch.bfloat16).cuda()
    W2 = (torch.randn(E, d, F, generator=gen) / d ** 0.5).to(torch.bfloat16).to(torch.float16).cuda()
    L = M.CapacityLayer(T, E, k, d, F)
    idx = torch.from_numpy(idx_h).cuda()
    gate = torch.full((T, k), 0.5, dtype=torch.float32, device="cuda")
    M.moe_histogram_maxvio(idx, E, 1, L.counts, L.loads, L.maxvio, L.balancedness, L.err)
    M.moe_capacity_ledger(L.counts, T, k, 5, 4, L.processed, L.overflow, L.padding, L.totals, L.err)
    M.moe_dispatch_capacity(x.cuda(), idx, L.counts, cap, L.workspace, L.recv, L.perm, L.src, L.err)
    M.moe_grouped_ffn_capacity(L.recv, W1, W3, W2, cap, L.h, L.y, L.err)
    M.moe_combine_capacity(L.y, L.perm, gate, L.out, L.err)
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    perm_ref, src_ref, rows = O.dispatch_capacity(idx_h, E, cap)
    assert L.processed.tolist() == g["processed"] == rows["processed"].tolist()
    assert L.overflow.tolist() == g["overflow"] and L.padding.tolist() == g["padding"]
    assert L.totals.tolist() == [5, 27, 5, 13]
    assert np.array_equal(L.perm.cpu().numpy(), perm_ref)
    assert np.array_equal(L.src.cpu().numpy(), src_ref)
    dropped = sorted((t, j) for t in range(T) for j in range(k) if L.perm[t, j].item() < 0)
    assert dropped == [(5, 0), (6, 0), (7, 0), (8, 0), (12, 0)]
    recv_ref = O.dispatch_padded(x.double().numpy(), src_ref)
    assert np.array_equal(to64(L.recv), recv_ref)
    y_ref = np.zeros((E * cap, d))
    for e in range(E):
        y_ref[e * cap:(e + 1) * cap] = O.expert_ffn(recv_ref[e * cap:(e + 1) * cap], to64(W1[e]),
                                                   to64(W3[e]), to64(W2[e]))
    assert_close_scaled(to64(L.y), y_ref, "y")
    out_ref = O.combine(y_ref, perm_ref, np.full((T, k), 0.5))
    assert_close_scaled(to64(L.out), out_ref, "out")


CASES = [(name, cf) for name in ("tiny", "near_balanced", "qwen_mv1", "mixtral", "deepseek")
         for cf in ((1, 1), (5, 4), (2, 1))]


@pytest.mark.parametrize("name,cf", CASES, ids=[f"{n}-cf{a}/{b}" for n, (a, b) in CASES])
def test_capacity_layer(name, cf):
    w = I.WORKLOADS[name]
    logits, x, weights = make_inputs(w)
    L = M.CapacityLayer(w.T, w.E, w.k, w.d, w.F, cf_num=cf[0], cf_den=cf[1])
    cap = L.cap
    assert cap == O.capacity_of(w.A, w.E, *cf)
    L.forward(logits.cuda(), x.cuda(), *weights)
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    idx, gate, err = O.topk_route(logits.numpy(), w.k)
    assert err == 0 and np.array_equal(L.idx.cpu().numpy(), idx)
    perm_ref, src_ref, rows = O.dispatch_capacity(idx, w.E, cap)
    led = O.capacity_ledger(rows["processed"] + rows["overflow"], w.A, w.E, *cf)
    assert L.totals.tolist() == [cap, int(led["processed"].sum()), int(led["overflow"].sum()),
                                 int(led["padding"].sum())]
    for key in ("processed", "overflow", "padding"):
        assert np.array_equal(getattr(L, key).cpu().numpy(), led[key]), key
    assert np.array_equal(L.perm.cpu().numpy(), perm_ref)
    assert np.array_equal(L.src.cpu().numpy(), src_ref)
    # recv: kept rows are the token rows bitwise, padding rows zero
    src_t = torch.from_numpy(src_ref.astype(np.int64)).cuda()
    keep = src_t >= 0
    xd = x.cuda()
    assert torch.equal(L.recv[keep], xd[src_t[keep]])
    assert int((L.recv[~keep] != 0).sum().item()) == 0
    E = w.E
    if w.T * w.d <= 4096 * 128:
        rows_chk = list(range(E * cap))
        tokens = list(range(w.T))
    else:
        # per sampled expert: the block's first rows, a tile boundary, its last kept row,
        # its first padding row and its last row
        rng = np.random.default_rng(17)
        experts = sorted(set(rng.choice(E, size=min(E, 6), replace=False).tolist()) |
                         {int(np.argmax(rows["processed"])), int(np.argmin(rows["processed"]))})
        rows_chk = []
        for e in experts:
            base, n = e * cap, int(rows["processed"][e])
            rows_chk += [base, base + 1, base + min(cap - 1, 127), base + min(cap - 1, 128)]
            rows_chk += [base + max(n - 1, 0), base + min(n, cap - 1), base + cap - 1]
        dropped_tok = sorted({t for t, j in zip(*np.nonzero(perm_ref < 0))})[:4]
        tokens = sorted(set(rng.choice(w.T, size=6, replace=False).tolist()) | set(dropped_tok)
                        | {w.T - 1})
    _check_rows(L, weights, E, cap, rows_chk, f"{name} cf {cf}")
    # out for the sampled tokens: their kept rows through the oracle's FFN
    need = sorted({int(r) for t in tokens for r in perm_ref[t] if r >= 0})
    _, y_need = _expert_rows_ref(_RowView({r: v for r, v in zip(
        need, to64(L.recv[torch.tensor(need, device="cuda")]))}) if need else _RowView({}),
        weights, E, cap, need)
    out_ref = O.combine(y_need, perm_ref, gate, tokens=tokens)
    out_gpu = to64(L.out[torch.tensor(tokens, device="cuda")])
    assert_close_scaled(out_gpu, np.stack([out_ref[t] for t in tokens]), f"out {name} cf {cf}")
    del L, weights
    torch.cuda.empty_cache()
