"""Test-side helpers: run the CUDA path through the binding, run the oracle on the same
seeded inputs, and compare.  Shares nothing with either side's arithmetic."""
from __future__ import annotations

import numpy as np
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import inputs as I
from oracle import moe_oracle as O

GATE_ATOL = 1e-6
FLOAT_RTOL = 1e-2  # |gpu - oracle| <= 1e-2 * max(1, |oracle|)


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close_scaled(gpu: np.ndarray, ref: np.ndarray, what: str):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    bound = FLOAT_RTOL * np.maximum(1.0, np.abs(ref))
    bad = np.abs(gpu - ref) > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements outside tolerance; "
                             f"first at {tuple(i)}: gpu {gpu[tuple(i)]} oracle {ref[tuple(i)]}")


def make_inputs(w: I.Workload, device="cuda"):
    logits = I.make_logits(w)
    x = I.make_x(w)
    W1, W3, W2 = I.make_weights(w, device=device)
    return logits, x, (W1, W3, W2)


def run_gpu(w: I.Workload, logits, x, weights, expert_to_rank=None, fused=False):
    """All seven calls in order on the current stream; returns the layer (buffers)."""
    W1, W3, W2 = weights
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F, fused=fused)
    lg = logits.to("cuda")
    xd = x.to("cuda")
    L.forward(lg, xd, W1, W3, W2)
    torch.cuda.synchronize()
    return L


def oracle_plan_fields(p, w: I.Workload):
    """The oracle's plan laid out field by field as the C ABI stores it."""
    R, S, E = w.R, w.S, w.E
    G = w.B + S
    groups = np.full((R, G, 4), -1, np.int64)
    n_groups = np.zeros(R, np.int64)
    for u, gl in enumerate(p["groups"]):
        n_groups[u] = len(gl)
        for i, g in enumerate(gl):
            groups[u, i] = g
    filled = [s for s in range(R * S) if p["replica_expert"][s] >= 0]
    rep_list = np.full(1 + R * S, -1, np.int64)
    rep_list[0] = len(filled)
    rep_list[1:1 + len(filled)] = filled
    return dict(kept_rows=np.array(p["kept_rows"]), room_prefix=np.array(p["room_prefix"]),
                expert_home_off=np.array(p["expert_home_off"]), stream_off=np.array(p["stream_off"]),
                replica_expert=np.array(p["replica_expert"]), replica_list=rep_list,
                n_groups=n_groups, groups=groups.reshape(-1))


def oracle_integer_path(w: I.Workload, logits: torch.Tensor):
    idx, gate, err = O.topk_route(logits.numpy(), w.k)
    h = O.expert_histogram(idx, w.E, w.R)
    p = O.plan_balanced(h["counts"], w.T, w.k, w.E, w.R, w.S)
    perm, src = O.permute(idx, p, w.E, w.R) if (err | h["err"] | p["err"]) == 0 else (None, None)
    return dict(idx=idx, gate=gate, err=err | h["err"] | p["err"], hist=h, plan=p, perm=perm, src=src)


def check_integer_parity(L, w: I.Workload, ref):
    assert int(L.err.item()) == ref["err"] == 0
    assert np.array_equal(L.idx.cpu().numpy(), ref["idx"]), "top-k ids"
    gdiff = np.abs(L.gate.cpu().double().numpy() - ref["gate"]).max() if w.T else 0.0
    assert gdiff <= GATE_ATOL, f"gate max abs diff {gdiff}"
    h = ref["hist"]
    assert np.array_equal(L.counts.cpu().numpy(), h["counts"]), "expert counts"
    assert np.array_equal(L.loads.cpu().numpy(), h["loads"]), "rank loads"
    assert L.maxvio.item() == h["maxvio"], ("maxvio", L.maxvio.item(), h["maxvio"])
    assert L.balancedness.item() == h["balancedness"]
    exp = oracle_plan_fields(ref["plan"], w)
    for name, v in exp.items():
        got = L.plan_field(name).cpu().numpy()
        assert np.array_equal(got, v), f"plan field {name}: gpu {got[:16]} oracle {v[:16]}"
    assert np.array_equal(L.perm.cpu().numpy(), ref["perm"]), "perm"
    assert np.array_equal(L.src.cpu().numpy(), ref["src"]), "src"


def check_rows_and_pool(L, w: I.Workload, x, weights, ref):
    """recv rows are bitwise token rows; pool slots are bitwise home experts."""
    xd = x.to("cuda")
    src = torch.from_numpy(ref["src"].astype(np.int64)).to("cuda")
    if w.T:
        assert torch.equal(L.recv, xd[src]), "recv rows"
    W1, W3, W2 = weights
    P1, P3, P2 = L.pool
    for slot, e in enumerate(ref["plan"]["replica_expert"]):
        if e >= 0:
            assert torch.equal(P1[slot], W1[e]) and torch.equal(P3[slot], W3[e]) and torch.equal(P2[slot], W2[e]), slot


def expert_weights64(weights, e):
    W1, W3, W2 = weights
    return to64(W1[e]), to64(W3[e]), to64(W2[e])


def check_ffn_combine_full(L, w, x, weights, ref):
    """Every row of h and y, every token of out, against the fp64 oracle."""
    p = ref["plan"]
    # the rows GEMM 1 reads: the dispatched copies, or (fused layer) the oracle's x[src]
    recv = to64(L.recv) if L.recv is not None else to64(x)[ref["src"]]
    cache = {}
    h_ref = np.zeros((w.A, w.F))
    y_ref = np.zeros((w.A, w.d))
    for gl in p["groups"]:
        for (r0, n, e, wref) in gl:
            if e not in cache:
                cache[e] = expert_weights64(weights, e)
            w1, w3, w2 = cache[e]  # a replica slot holds the home weights bitwise
            X = recv[r0:r0 + n]
            hh = O.silu(X @ w1.T) * (X @ w3.T)
            h_ref[r0:r0 + n] = hh
            y_ref[r0:r0 + n] = O.expert_ffn(X, w1, w3, w2)
    assert_close_scaled(to64(L.h), h_ref, "h")
    assert_close_scaled(to64(L.y), y_ref, "y")
    out_ref = O.combine(y_ref, ref["perm"], ref["gate"])
    assert_close_scaled(to64(L.out), out_ref, "out")
    # combine in isolation: the GPU's own y and gates through the oracle's combine
    out_iso = O.combine(to64(L.y), L.perm.cpu().numpy(), L.gate.cpu().double().numpy())
    assert_close_scaled(to64(L.out), out_iso, "out (combine alone)")


def check_ffn_combine_sampled(L, w, x, weights, ref, tokens):
    """Sampled tokens: all k rows of each through the oracle FFN, then its combine."""
    p = ref["plan"]
    row_group = {}
    want = set()
    for t in tokens:
        for j in range(w.k):
            want.add(int(ref["perm"][t, j]))
    for gl in p["groups"]:
        for (r0, n, e, wref) in gl:
            for r in want:
                if r0 <= r < r0 + n:
                    row_group[r] = e
    rows = sorted(want)
    if L.recv is not None:
        recv = to64(L.recv[torch.tensor(rows, device="cuda")])
    else:
        recv = to64(x)[ref["src"][rows]]
    ridx = {r: i for i, r in enumerate(rows)}
    y_ref = {}
    by_e = {}
    for r in rows:
        by_e.setdefault(row_group[r], []).append(r)
    for e, rs in by_e.items():
        w1, w3, w2 = expert_weights64(weights, e)
        X = recv[[ridx[r] for r in rs]]
        ys = O.expert_ffn(X, w1, w3, w2)
        for r, yr in zip(rs, ys):
            y_ref[r] = yr
    y_gpu = to64(L.y[torch.tensor(rows, device="cuda")])
    assert_close_scaled(y_gpu, np.stack([y_ref[r] for r in rows]), "y (sampled rows)")
    out_ref = O.combine(y_ref, ref["perm"], ref["gate"], tokens=tokens)
    out_gpu = to64(L.out[torch.tensor(tokens, device="cuda")])
    assert_close_scaled(out_gpu, np.stack([out_ref[t] for t in tokens]), "out (sampled tokens)")


def edge_rows(plan, E: int, tile: int = 128):
    """Rows of the grouped FFN where a tiling mistake would show, as {name: [rows]}: every
    row of the last (partial) tile of the largest group; rows 126-129 of a group that spans
    more than one tile (the first tile boundary); every row of the smallest replica group
    (weights from a pool slot); every row of the last group of the last rank."""
    groups = [g for gl in plan["groups"] for g in gl]
    out = {}
    r0, n, _, _ = max(groups, key=lambda g: (g[1], -g[0]))
    last = r0 + tile * ((n - 1) // tile)
    out["last tile of the largest group"] = list(range(last, r0 + n))
    multi = [g for g in groups if g[1] > tile + 2]
    if multi:
        r0, n, _, _ = multi[0]
        out["rows 126-129 of a multi-tile group"] = [r0 + i for i in range(tile - 2, tile + 2)]
    reps = [g for g in groups if g[3] >= E]
    if reps:
        r0, n, _, _ = min(reps, key=lambda g: (g[1], g[0]))
        out["smallest replica group"] = list(range(r0, r0 + n))
    lastr = [gl for gl in plan["groups"] if gl][-1]
    r0, n, _, _ = lastr[-1]
    out["last group of the last rank"] = list(range(r0, r0 + n))
    return out


def check_ffn_edge_rows(L, w, x, weights, ref):
    """h and y of edge_rows() against the fp64 oracle (each row through its group's expert;
    a replica slot holds its expert's home weights bitwise)."""
    p = ref["plan"]
    row_expert = {}
    sets = edge_rows(p, w.E)
    want = sorted({r for rs in sets.values() for r in rs})
    wanted = set(want)
    for gl in p["groups"]:
        for (r0, n, e, _) in gl:
            for r in range(r0, r0 + n):
                if r in wanted:
                    row_expert[r] = e
    rows_t = torch.tensor(want, device="cuda")
    if L.recv is not None:
        recv = to64(L.recv[rows_t])
    else:
        recv = to64(x)[ref["src"][want]]
    ridx = {r: i for i, r in enumerate(want)}
    h_ref = np.zeros((len(want), w.F))
    y_ref = np.zeros((len(want), w.d))
    by_e = {}
    for r in want:
        by_e.setdefault(row_expert[r], []).append(r)
    for e, rs in by_e.items():
        w1, w3, w2 = expert_weights64(weights, e)
        X = recv[[ridx[r] for r in rs]]
        ii = [ridx[r] for r in rs]
        h_ref[ii] = O.silu(X @ w1.T) * (X @ w3.T)
        y_ref[ii] = O.expert_ffn(X, w1, w3, w2)
    h_gpu = to64(L.h[rows_t])
    y_gpu = to64(L.y[rows_t])
    for name, rs in sets.items():
        ii = [ridx[r] for r in rs]
        assert_close_scaled(h_gpu[ii], h_ref[ii], f"h, {name}")
        assert_close_scaled(y_gpu[ii], y_ref[ii], f"y, {name}")
    return sets
