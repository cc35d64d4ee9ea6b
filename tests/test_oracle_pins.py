"""Pins of the CPU oracle against what the pages and plain mathematics fix (no GPU).

Each check is independent of the oracle's own code path: printed values of the worked
fixture, brute-force enumeration on tiny inputs, closed forms and invariants.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hotspot_fixture.json")


@pytest.fixture(scope="module")
def fx():
    with open(GOLD) as f:
        g = json.load(f)
    idx = np.array([[int(p[0]), int(p[1])] for p in g["pairs"]], dtype=np.int32)
    origin = np.arange(g["tokens"]) % g["ranks"]
    return g, idx, origin


def _mapping(groups, E):
    m = np.zeros(E, dtype=np.int64)
    for r, g in enumerate(groups):
        for e in g:
            m[e] = r
    return m


# ----------------------------------------------------------- the pages' worked fixture
def test_fixture_demand_and_balancedness(fx):
    g, idx, _ = fx
    E, R = g["experts"], g["ranks"]
    assert idx.size == g["assignments"] == g["tokens"] * g["top_k"]
    h = O.expert_histogram(idx, E, R)
    assert h["err"] == 0
    assert list(h["counts"]) == g["expert_demand"]
    num, den = g["expert_balancedness_num_den"]
    assert h["expert_balancedness"] == float(Fraction(num, den))
    assert h["counts"].sum() / E == g["expert_mean"]


def test_fixture_rank_demand_two_mappings(fx):
    g, idx, _ = fx
    E, R = g["experts"], g["ranks"]
    m0 = _mapping(g["initial_mapping"], E)
    m1 = _mapping(g["proposed_mapping"], E)
    # the initial mapping is the contiguous home map
    assert list(m0) == list(O.home_rank_map(E, R))
    h0 = O.expert_histogram(idx, E, R, m0)
    h1 = O.expert_histogram(idx, E, R, m1)
    assert list(h0["loads"]) == g["initial_rank_demand"]
    assert list(h1["loads"]) == g["proposed_rank_demand"]
    num, den = g["initial_balancedness_num_den"]
    assert h0["balancedness"] == float(Fraction(num, den))
    assert round(h0["balancedness"], 6) == g["initial_balancedness_printed"]
    assert h1["balancedness"] == g["proposed_balancedness"]
    # maxvio = (max - mean)/mean: 15/8 - 1 and 10/8 - 1
    assert h0["maxvio"] == 0.875 and h1["maxvio"] == 0.25
    assert h0["expert_maxvio"] == 1.25


def test_fixture_capacity_ledger(fx):
    g, idx, _ = fx
    h = O.expert_histogram(idx, g["experts"], g["ranks"])
    num, den = g["capacity_factor_num_den"]
    led = O.capacity_ledger(h["counts"], g["assignments"], g["experts"], num, den)
    assert led["cap"] == g["capacity"]
    assert list(led["processed"]) == g["processed"] and led["processed"].sum() == g["processed_sum"]
    assert list(led["overflow"]) == g["overflow"] and led["overflow"].sum() == g["overflow_sum"]
    assert list(led["padding"]) == g["padding"] and led["padding"].sum() == g["padding_sum"]


def test_fixture_remote_routes(fx):
    g, idx, origin = fx
    E = g["experts"]
    r0 = O.remote_routes(idx, origin, _mapping(g["initial_mapping"], E))
    r1 = O.remote_routes(idx, origin, _mapping(g["proposed_mapping"], E))
    assert r0 == g["remote_initial"] and r0 / g["assignments"] == g["remote_initial_share"]
    assert r1 == g["remote_proposed"] and r1 / g["assignments"] == g["remote_proposed_share"]


def test_fixture_validation_rules(fx):
    g, idx, _ = fx
    bad = idx.copy()
    bad[3, 1] = bad[3, 0]          # token repeats an expert
    assert O.expert_histogram(bad, 8, 4)["err"] & O.ERR_DUPLICATE
    bad = idx.copy()
    bad[5, 0] = 8                  # unknown expert
    assert O.expert_histogram(bad, 8, 4)["err"] & O.ERR_ID_RANGE
    bad[5, 0] = -1
    assert O.expert_histogram(bad, 8, 4)["err"] & O.ERR_ID_RANGE


def test_fixture_mapping_must_cover_every_expert(fx):
    """"If any expert is missing from a mapping, stop": a rank outside [0, R) leaves an
    expert with no owner.  The fixture's initial mapping {0,1},{2,3},{4,5},{6,7} gives
    rank demand [15,9,5,3]; with expert 7 (demand 1) unmapped (-1) no rank may receive
    its assignment -- [15,9,5,2], not [15,9,5,3] with rank 3 wrapping round -- and with
    expert 0 (demand 9) mapped to rank 4 = R the demand is [6,9,5,3].  Both set error
    bit 2 and nothing else; the expert counts stay [9,6,5,4,3,2,2,1]."""
    g, idx, _ = fx
    E, R = g["experts"], g["ranks"]
    m = _mapping(g["initial_mapping"], E)
    assert O.expert_histogram(idx, E, R, m)["err"] == 0
    for e, r, loads in ((7, -1, [15, 9, 5, 2]), (0, R, [6, 9, 5, 3]), (3, -R, [15, 5, 5, 3])):
        bad = m.copy()
        bad[e] = r
        h = O.expert_histogram(idx, E, R, bad)
        assert h["err"] == O.ERR_ID_RANGE
        assert list(h["loads"]) == loads
        assert list(h["counts"]) == g["expert_demand"]


def test_fixture_fixed_capacity_dispatch(fx):
    """Fixed capacity 5 on the fixture ("Make expert capacity, overflow, and padding
    explicit"): processed [5,5,5,4,3,2,2,1] (27), overflow [4,1,0,...] (5), padding 13.
    Derived by hand from the pairs 01,02,03,04,05,06,07,01,02,12,12,12,13,34,34,56 with
    each expert keeping its first five assignments in token order: expert 0 is chosen by
    tokens 0..8 and keeps 0..4 (tokens 5,6,7,8 dropped); expert 1 by tokens 0,7,9,10,11,12
    and drops token 12; expert 2 by 1,8,9,10,11 (all kept); expert 3 by 2,12,13,14 (one
    padding row)."""
    g, idx, _ = fx
    E = g["experts"]
    cap = O.capacity_of(g["assignments"], E, *g["capacity_factor_num_den"])
    assert cap == g["capacity"] == 5
    perm, src, rows = O.dispatch_capacity(idx, E, cap)
    assert list(rows["processed"]) == g["processed"] and rows["processed"].sum() == 27
    assert list(rows["overflow"]) == g["overflow"] and rows["overflow"].sum() == 5
    assert list(rows["padding"]) == g["padding"] and rows["padding"].sum() == 13
    dropped = sorted((t, j) for t in range(16) for j in range(2) if perm[t, j] < 0)
    assert dropped == [(5, 0), (6, 0), (7, 0), (8, 0), (12, 0)]
    assert list(src[0:5]) == [0, 1, 2, 3, 4]
    assert list(src[5:10]) == [0, 7, 9, 10, 11]
    assert list(src[10:15]) == [1, 8, 9, 10, 11]
    assert list(src[15:20]) == [2, 12, 13, 14, -1]
    assert int((src < 0).sum()) == 13
    # every kept assignment is the row its block says; rows of one expert hold that expert
    for t in range(16):
        for j in range(2):
            r = int(perm[t, j])
            if r >= 0:
                assert src[r] == t and r // cap == idx[t, j]


def test_capacity_ledger_invariants_on_random_traces():
    """On random traces and capacities: processed + overflow = demand, processed +
    padding = cap, kept assignments fill each block from its first row with no gaps, and
    the dispatch's counts equal capacity_ledger's (two separate restatements of the page's
    min / max formulas)."""
    rng = np.random.default_rng(3)
    for _ in range(40):
        E = int(rng.integers(1, 9))
        k = int(rng.integers(1, E + 1))
        T = int(rng.integers(0, 30))
        idx = np.array([rng.permutation(E)[:k] for _ in range(T)], dtype=np.int32).reshape(T, k)
        num, den = int(rng.integers(1, 9)), int(rng.integers(1, 5))
        cap = O.capacity_of(T * k, E, num, den)
        perm, src, rows = O.dispatch_capacity(idx, E, cap)
        demand = np.bincount(idx.reshape(-1), minlength=E) if T else np.zeros(E, int)
        assert np.array_equal(rows["processed"] + rows["overflow"], demand)
        assert np.array_equal(rows["processed"] + rows["padding"], np.full(E, cap))
        led = O.capacity_ledger(demand, T * k, E, num, den)
        assert led["cap"] == cap
        for key in ("processed", "overflow", "padding"):
            assert np.array_equal(led[key], rows[key])
        for e in range(E):
            block = src[e * cap:(e + 1) * cap]
            n = int(rows["processed"][e])
            assert (block[:n] >= 0).all() and (block[n:] == -1).all()
        assert int((perm >= 0).sum()) == int(rows["processed"].sum())


def test_capacity_above_every_demand_is_the_dropless_layer():
    """With a capacity factor large enough that no expert overflows, the fixed-capacity
    layer computes the dropless layer's output (different row layout, same sums)."""
    rng = np.random.default_rng(4)
    T, E, k, d, F = 24, 4, 2, 16, 24
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = rng.standard_normal((T, d))
    W1 = rng.standard_normal((E, F, d)) / 4
    W3 = rng.standard_normal((E, F, d)) / 4
    W2 = rng.standard_normal((E, d, F)) / 4
    ref = O.layer(logits, x, W1, W3, W2, k, 2, 2)
    cap = O.layer_capacity(logits, x, W1, W3, W2, k, cf_num=E, cf_den=1)
    assert ref["err"] == 0 and cap["err"] == 0
    assert (cap["perm"] >= 0).all() and cap["rows"]["overflow"].sum() == 0
    assert np.allclose(cap["out"], ref["out"], rtol=1e-12, atol=1e-12)
    # and a small factor drops assignments: those tokens lose the dropped terms
    tight = O.layer_capacity(logits, x, W1, W3, W2, k, cf_num=1, cf_den=2)
    assert tight["rows"]["overflow"].sum() > 0
    assert not np.allclose(tight["out"], ref["out"])


def test_combine_leaves_dropped_assignments_out():
    """Identity experts (y = the dispatched rows) on a fixed-capacity buffer: token t gets
    (sum of its kept gates) * x_t -- the dropped choices add nothing -- and a token with
    every choice dropped gets zeros."""
    rng = np.random.default_rng(5)
    T, E, k, d = 40, 4, 2, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[:, 0] += 3.0  # expert 0 overflows
    x = rng.standard_normal((T, d))
    idx, gate, _ = O.topk_route(logits, k)
    cap = O.capacity_of(T * k, E, 1, 1)
    perm, src, rows = O.dispatch_capacity(idx, E, cap)
    assert rows["overflow"][0] > 0
    y = O.dispatch_padded(x, src)
    y[src < 0] = 1e3  # no kept assignment points at a padding row: its contents never show
    out = O.combine(y, perm, gate)
    kept = np.where(perm >= 0, gate, 0.0).sum(axis=1)
    assert np.allclose(out, kept[:, None] * x, rtol=1e-13, atol=1e-13)
    none = O.combine(np.zeros((4, d)), np.full((3, 2), -1), np.full((3, 2), 0.5))
    assert none.shape == (3, d) and (none == 0).all()


def test_fixture_plan_derived_by_hand(fx):
    """The balanced plan of the fixture at R=4, S=2, derived by hand from the plan's
    steps: C = 8; rank 0 keeps e1 (6) and streams e0 (9): room 2; rank 1 keeps e3 (4),
    streams e2 (5): room 4; rank 2 keeps e5, e4 (2+3): room 3; rank 3 keeps e7, e6 (1+2):
    room 5.  Stream [e0 x9, e2 x5] cut by rooms [2,4,3,5]: e0 tokens {0,1} stay home,
    {2..5} go to rank 1, {6,7,8} to rank 2; e2 tokens {1,8,9,10,11} go to rank 3."""
    g, idx, _ = fx
    counts = O.expert_histogram(idx, 8, 4)["counts"]
    p = O.plan_balanced(counts, 16, 2, 8, 4, 2)
    assert p["err"] == 0 and p["C"] == 8
    assert p["kept_rows"] == [6, 4, 5, 3]
    assert p["room_prefix"] == [0, 2, 6, 9, 14]
    assert p["expert_home_off"] == [-1, 0, -1, 0, 0, 3, 0, 2]
    assert p["stream_off"] == [0, 9, 9, 14, 14, 14, 14, 14, 14]
    assert p["replica_expert"] == [-1, -1, 0, -1, 0, -1, 2, -1]
    assert p["groups"] == [
        [(0, 6, 1, 1), (6, 2, 0, 0)],
        [(8, 4, 3, 3), (12, 4, 0, 8 + 1 * 2 + 0)],
        [(16, 3, 4, 4), (19, 2, 5, 5), (21, 3, 0, 8 + 2 * 2 + 0)],
        [(24, 2, 6, 6), (26, 1, 7, 7), (27, 5, 2, 8 + 3 * 2 + 0)],
    ]
    perm, src = O.permute(idx, p, 8, 4)
    e0_tokens = [t for t in range(16) if 0 in idx[t]]
    assert e0_tokens == list(range(9))
    rows_e0 = [int(perm[t][list(idx[t]).index(0)]) for t in e0_tokens]
    assert rows_e0 == [6, 7, 12, 13, 14, 15, 21, 22, 23]
    e2_tokens = [t for t in range(16) if 2 in idx[t]]
    assert e2_tokens == [1, 8, 9, 10, 11]
    assert [int(perm[t][list(idx[t]).index(2)]) for t in e2_tokens] == [27, 28, 29, 30, 31]
    # S = 0 cannot hold the three replicas
    assert O.plan_balanced(counts, 16, 2, 8, 4, 0)["err"] == O.ERR_SLOTS


# ----------------------------------------------------------- top-k: brute force
def _topk_bruteforce(row, k):
    """Rank of expert e = #experts with a larger logit + #lower ids with an equal one."""
    E = len(row)
    rank = [sum(1 for f in range(E) if row[f] > row[e] or (row[f] == row[e] and f < e))
            for e in range(E)]
    return [rank.index(r) for r in range(k)]


def test_topk_bruteforce_with_ties():
    rng = np.random.default_rng(1)
    for E in (1, 2, 3, 5, 8):
        for k in range(1, E + 1):
            # values from a small set force many exact ties; include +0 and -0
            vals = np.array([-1.0, -0.0, 0.0, 0.5, 2.0], dtype=np.float32)
            logits = vals[rng.integers(0, len(vals), size=(20, E))]
            idx, gate, err = O.topk_route(logits, k)
            assert err == 0
            for t in range(20):
                assert list(idx[t]) == _topk_bruteforce(logits[t].astype(np.float64), k)
                assert abs(gate[t].sum() - 1.0) < 1e-15 and (gate[t] >= 0).all()


def test_topk_special_cases():
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((30, 7)).astype(np.float32)
    # k = 1: lowest-index argmax, gate exactly 1
    idx, gate, _ = O.topk_route(logits, 1)
    assert list(idx[:, 0]) == [int(np.argmax(r)) for r in logits]
    assert (gate == 1.0).all()
    # k = E: a full descending ordering
    idx, gate, _ = O.topk_route(logits, 7)
    for t in range(30):
        assert sorted(idx[t]) == list(range(7))
        assert all(logits[t, idx[t, j]] >= logits[t, idx[t, j + 1]] for j in range(6))
    # k = 2: gate_0 = sigmoid(l0 - l1)
    idx, gate, _ = O.topk_route(logits, 2)
    for t in range(30):
        l0, l1 = float(logits[t, idx[t, 0]]), float(logits[t, idx[t, 1]])
        assert abs(gate[t, 0] - 1.0 / (1.0 + math.exp(l1 - l0))) < 1e-15
    # equal logits: ids 0..k-1, gates 1/k
    idx, gate, _ = O.topk_route(np.zeros((3, 6), np.float32), 4)
    assert (idx == np.arange(4)).all() and np.allclose(gate, 0.25, atol=0, rtol=0)


def test_topk_nonfinite_sets_error():
    for bad in (np.nan, np.inf, -np.inf):
        logits = np.zeros((4, 5), np.float32)
        logits[2, 3] = bad
        assert O.topk_route(logits, 2)[2] == O.ERR_NONFINITE


# ----------------------------------------------------------- imbalance identities
def test_maxvio_identities():
    rng = np.random.default_rng(3)
    for _ in range(50):
        E, R, k = 8, 4, 3
        T = int(rng.integers(1, 12))
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        h = O.expert_histogram(idx, E, R)
        A = T * k
        assert h["loads"].sum() == A == h["counts"].sum()
        assert abs(h["maxvio"] - (1.0 / h["balancedness"] - 1.0)) < 1e-12
        assert h["maxvio"] == float(Fraction(R * int(h["loads"].max()) - A, A))
    # perfectly balanced: every rank gets the same load -> 0; all on one rank -> R-1
    idx = np.array([[0, 2], [4, 6], [1, 3], [5, 7]], np.int32)
    assert O.expert_histogram(idx, 8, 4)["maxvio"] == 0.0
    idx = np.array([[0, 1]] * 5, np.int32)
    assert O.expert_histogram(idx, 8, 4)["maxvio"] == 3.0
    # empty trace
    h = O.expert_histogram(np.zeros((0, 2), np.int32), 8, 4)
    assert h["maxvio"] == 0.0 and h["balancedness"] == 1.0


# ----------------------------------------------------------- plan: exhaustive invariants
def _check_plan_invariants(idx, E, R, S):
    T, k = idx.shape
    counts = np.bincount(idx.ravel(), minlength=E) if idx.size else np.zeros(E, int)
    p = O.plan_balanced(counts, T, k, E, R, S)
    C = T * k // R
    B = E // R
    perm, src = O.permute(idx, p, E, R)
    # every assignment placed exactly once; every rank exactly C rows
    rows = sorted(int(r) for r in perm.ravel())
    assert rows == list(range(R * C))
    for t in range(T):
        for j in range(k):
            assert src[perm[t, j]] == t
    # a group table tiles each rank's rows and names the expert of each row
    row_expert = {}
    for t in range(T):
        for j in range(k):
            row_expert[int(perm[t, j])] = int(idx[t, j])
    # independent replica count: (rank, expert) pairs of assignments placed away from home
    away = {}
    for r, e in row_expert.items():
        u = r // C
        if e // B != u:
            away.setdefault(u, set()).add(e)
    need = max((len(v) for v in away.values()), default=0)
    assert (p["err"] == O.ERR_SLOTS) == (need > S)
    if p["err"]:
        return
    for u in range(R):
        covered = []
        for (r0, n, e, ref) in p["groups"][u]:
            assert n > 0 and u * C <= r0 and r0 + n <= (u + 1) * C
            for r in range(r0, r0 + n):
                assert row_expert[r] == e
            covered += list(range(r0, r0 + n))
            if e // B == u:
                assert ref == e
            else:
                assert E <= ref < E + R * S and (ref - E) // S == u
                assert p["replica_expert"][ref - E] == e
        assert sorted(covered) == list(range(u * C, (u + 1) * C))
        reps = [ref for (_, _, e, ref) in p["groups"][u] if ref >= E]
        assert len(reps) == len(away.get(u, ())) <= S
    # kept experts are whole at home
    for e in range(E):
        if p["kept"][e]:
            assert all(r // C == e // B for r, ee in row_expert.items() if ee == e)


def test_plan_invariants_exhaustive_tiny():
    E, k = 4, 2
    pairs = [list(p) for p in itertools.permutations(range(E), k)]
    n = 0
    for T in (1, 2, 3, 4):
        for combo in itertools.product(range(len(pairs)), repeat=T):
            idx = np.array([pairs[c] for c in combo], np.int32)
            for R in (1, 2, 4):
                if (T * k) % R:
                    continue
                for S in (0, 1, 2):
                    _check_plan_invariants(idx, E, R, S)
                    n += 1
    assert n > 10000


def test_plan_invariants_random_larger():
    rng = np.random.default_rng(4)
    for _ in range(40):
        E, R = 16, 4
        k = int(rng.integers(1, 5))
        T = 4 * int(rng.integers(1, 10))
        alpha = float(rng.uniform(0, 3))
        w = np.exp(-alpha * np.log(np.arange(E) + 1.0))
        idx = np.stack([rng.choice(E, size=k, replace=False, p=w / w.sum()) for _ in range(T)]).astype(np.int32)
        for S in (0, 1, 2, 4):
            _check_plan_invariants(idx, E, R, S)


# ----------------------------------------------------------- dispatch / prefetch
def test_dispatch_prefetch_identities():
    rng = np.random.default_rng(5)
    E, R, k, T, S, d, F = 8, 4, 2, 12, 2, 4, 6
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    idx[:8, 0] = 0  # make expert 0 hot
    for t in range(8):
        if idx[t, 1] == 0:
            idx[t, 1] = 1
    counts = np.bincount(idx.ravel(), minlength=E)
    p = O.plan_balanced(counts, T, k, E, R, S)
    assert p["err"] == 0
    x = rng.standard_normal((T, d))
    perm, src = O.permute(idx, p, E, R)
    recv = O.dispatch(x, src)
    for t in range(T):
        for j in range(k):
            assert (recv[perm[t, j]] == x[t]).all()
    W1, W3, W2 = (rng.standard_normal(s) for s in ((E, F, d), (E, F, d), (E, d, F)))
    pool = O.prefetch(p, W1, W3, W2, R, S)
    assert len(pool) == sum(1 for e in p["replica_expert"] if e >= 0) > 0
    for slot, (a, b, c) in pool.items():
        e = p["replica_expert"][slot]
        assert (a == W1[e]).all() and (b == W3[e]).all() and (c == W2[e]).all()


# ----------------------------------------------------------- FFN closed forms
SILU_1 = 0.7310585786300049  # logistic(1) = e / (1 + e)


def test_ffn_closed_forms():
    assert abs(SILU_1 - math.e / (1.0 + math.e)) < 1e-16
    # identity weights: y_i = silu(x_i) * x_i
    I = np.eye(4)
    x = np.array([[1.0, 0.0, -1.0, 2.0]])
    y = O.expert_ffn(x, I, I, I)
    expect = [SILU_1, 0.0, -(1 - SILU_1) * -1.0, 2.0 * 2.0 / (1.0 + math.exp(-2.0))]
    assert np.allclose(y[0], expect, rtol=0, atol=1e-15)
    # single-entry, non-square weights: a transposed or dropped operand lands elsewhere
    d, F = 2, 3
    w1 = np.zeros((F, d)); w1[2, 1] = 1.0     # g_2 = x_1
    w3 = np.zeros((F, d)); w3[2, 0] = 1.0     # u_2 = x_0
    w2 = np.zeros((d, F)); w2[1, 2] = 1.0     # y_1 = h_2
    y = O.expert_ffn(np.array([[2.0, 1.0]]), w1, w3, w2)
    assert y[0, 0] == 0.0 and abs(y[0, 1] - 2.0 * SILU_1) < 1e-15
    # silu is odd-symmetric around its sigmoid: silu(-z) = silu(z) - z
    z = np.linspace(-5, 5, 11)
    assert np.allclose(O.silu(-z), O.silu(z) - z, atol=1e-14, rtol=0)


# ----------------------------------------------------------- combine / whole layer
def test_combine_identity_and_scaled_experts():
    rng = np.random.default_rng(6)
    E, R, k, T, S, d = 8, 4, 3, 8, 2, 5
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[:, 0] += 3.0
    x = rng.standard_normal((T, d))
    idx, gate, _ = O.topk_route(logits, k)
    counts = np.bincount(idx.ravel(), minlength=E)
    p = O.plan_balanced(counts, T, k, E, R, S)
    assert p["err"] == 0
    perm, src = O.permute(idx, p, E, R)
    recv = O.dispatch(x, src)
    out = O.combine(recv, perm, gate)       # identity experts
    assert np.allclose(out, x, atol=1e-14, rtol=0)
    c = rng.uniform(0.5, 2.0, size=E)
    row_e = np.zeros(R * p["C"], int)
    for t in range(T):
        for j in range(k):
            row_e[perm[t, j]] = idx[t, j]
    y = recv * c[row_e][:, None]
    out = O.combine(y, perm, gate)
    expect = np.stack([sum(gate[t, j] * c[idx[t, j]] for j in range(k)) * x[t] for t in range(T)])
    assert np.allclose(out, expect, atol=1e-14, rtol=0)


def test_layer_identity_experts_returns_x():
    """Whole path on the tiny shape with every expert's weights the identity: each
    expert computes silu(x)*x and the gates sum to one, so the layer returns silu(x)*x."""
    rng = np.random.default_rng(7)
    T, E, k, R, S, d = 16, 8, 2, 4, 2, 4
    logits = rng.standard_normal((T, E)).astype(np.float32) - 1.5 * np.log(np.arange(E) + 1.0)
    x = rng.standard_normal((T, d))
    I = np.stack([np.eye(d)] * E)
    res = O.layer(logits, x, I, I, I, k, R, S)
    assert res["err"] == 0
    ref = O.silu(x) * x      # every expert computes silu(x)*x, gates sum to one
    assert np.allclose(res["out"], ref, atol=1e-13, rtol=0)


# ----------------------------------------------------------- bias-only selection
def test_biased_topk_pins():
    rng = np.random.default_rng(20)
    logits = rng.standard_normal((40, 12)).astype(np.float32)
    # zero bias is plain top-k
    i0, g0, _ = O.topk_route(logits, 3)
    i1, g1, _ = O.topk_route_biased(logits, np.zeros(12, np.float32), 3)
    assert (i0 == i1).all() and np.array_equal(g0, g1)
    # a large bias on experts {2, 7} forces them into every token's choice
    bias = np.zeros(12, np.float32)
    bias[[2, 7]] = 100.0
    idx, gate, err = O.topk_route_biased(logits, bias, 2)
    assert err == 0
    for t in range(40):
        assert sorted(idx[t]) == [2, 7]
        # the gate ignores the bias: softmax of the two unbiased logits, in chosen order
        a, b = float(logits[t, idx[t, 0]]), float(logits[t, idx[t, 1]])
        assert abs(gate[t, 0] - 1.0 / (1.0 + math.exp(b - a))) < 1e-15
    # order follows the biased score: 7 leads where logit7 + 100 > logit2 + 100
    for t in range(40):
        first = 7 if np.float32(logits[t, 7] + np.float32(100)) > np.float32(logits[t, 2] + np.float32(100)) else 2
        assert idx[t, 0] == first or logits[t, 7] + 100 == logits[t, 2] + 100
    # unequal biases on the chosen pair: a gate computed from the biased scores would be
    # shifted by the bias difference; the gate must stay the softmax of the raw logits
    bias2 = np.zeros(12, np.float32)
    bias2[2], bias2[7] = 100.0, 101.5
    idx, gate, err = O.topk_route_biased(logits, bias2, 2)
    assert err == 0
    for t in range(40):
        assert sorted(idx[t]) == [2, 7]
        a, b = float(logits[t, idx[t, 0]]), float(logits[t, idx[t, 1]])
        assert abs(gate[t, 0] - 1.0 / (1.0 + math.exp(b - a))) < 1e-15
    bad = bias.copy()
    bad[3] = np.nan
    assert O.topk_route_biased(logits, bad, 2)[2] == O.ERR_NONFINITE


# ----------------------------------------------------------- expert parallelism
def _ep_case(seed, W, T, E, k, d=8, F=12, skew=1.0):
    rng = np.random.default_rng(seed)
    logits = (rng.standard_normal((W * T, E)) - skew * np.log(np.arange(E) + 1.0)).astype(np.float32)
    x = rng.standard_normal((W * T, d))
    W1 = rng.standard_normal((E, F, d)) / 3
    W3 = rng.standard_normal((E, F, d)) / 3
    W2 = rng.standard_normal((E, d, F)) / 3
    return logits, x, W1, W3, W2


EP_CASES = [(0, 1, 12, 4, 2, 2), (1, 2, 12, 8, 2, 4), (2, 4, 6, 8, 2, 4), (3, 3, 8, 6, 3, 4),
            (4, 4, 16, 16, 4, 8)]


def test_ep_layer_is_the_layer_of_the_rank_major_batch():
    """W processes, each routing its own T tokens, compute the undistributed layer of the
    concatenated batch (rank u's token t = job token u*T + t) with R = W: the same rows in
    the same places, every rank exactly C rows, the same outputs."""
    for seed, W, T, E, k, S in EP_CASES:
        logits, x, W1, W3, W2 = _ep_case(seed, W, T, E, k)
        ep = O.ep_layer(np.split(logits, W), np.split(x, W), W1, W3, W2, k, S)
        ref = O.layer(logits, x, W1, W3, W2, k, W, S)
        assert ep["err"] == 0 and ref["err"] == 0
        C = ref["plan"]["C"]
        perm = np.concatenate([r["perm"] for r in ep["ranks"]])
        assert np.array_equal(perm, ref["perm"])
        assert sorted(perm.ravel().tolist()) == list(range(W * C))  # every rank: C rows
        for u, r in enumerate(ep["ranks"]):
            assert np.array_equal(r["recv"], ref["recv"][u * C:(u + 1) * C])
            assert np.allclose(r["y"], ref["y"][u * C:(u + 1) * C], rtol=1e-12, atol=1e-12)
        out = np.concatenate([r["out"] for r in ep["ranks"]])
        assert np.allclose(out, ref["out"], rtol=1e-12, atol=1e-12)


def test_ep_rank_base_counts_the_lower_ranks_assignments():
    """q_base of rank u and expert e is the number of assignments of e made by the job's
    tokens before u*T, counted directly on the concatenated batch."""
    for seed, W, T, E, k, S in EP_CASES:
        logits, *_ = _ep_case(seed, W, T, E, k)
        idx = O.topk_route(logits, k)[0]
        shards = np.split(idx, W)
        counts_all = np.stack([O.ep_local_counts(s, E)[0] for s in shards])
        for u in range(W):
            direct = [int((idx[:u * T] == e).sum()) for e in range(E)]
            assert O.ep_rank_base(counts_all, u).tolist() == direct


def test_ep_error_bits_reach_every_rank():
    """A non-finite logit on one rank, or a repeated expert in one rank's trace, is an
    error of the whole job (every rank computes the plan from the exchanged counts)."""
    logits, x, W1, W3, W2 = _ep_case(5, 2, 8, 8, 2)
    bad = logits.copy()
    bad[11, 3] = np.nan  # rank 1's token 3
    ep = O.ep_layer(np.split(bad, 2), np.split(x, 2), W1, W3, W2, 2, 4)
    assert ep["err"] & O.ERR_NONFINITE
    c, e = O.ep_local_counts(np.array([[1, 1], [0, 9]]), 8)
    assert e == O.ERR_DUPLICATE | O.ERR_ID_RANGE and c.tolist() == [1, 2, 0, 0, 0, 0, 0, 0]


def test_ep_backward_is_the_backward_of_the_rank_major_batch():
    """The W-process backward -- dy written across ranks, each rank's groups on its own rows,
    replica gradients reduced to the home rank -- equals layer_backward() of the
    concatenated batch: dx, dlogits and every weight gradient."""
    for seed, W, T, E, k, S in EP_CASES:
        logits, x, W1, W3, W2 = _ep_case(seed, W, T, E, k)
        rng = np.random.default_rng(100 + seed)
        dout = rng.standard_normal(x.shape)
        ep = O.ep_layer(np.split(logits, W), np.split(x, W), W1, W3, W2, k, S)
        ebw = O.ep_layer_backward(ep, np.split(dout, W), W1, W3, W2, E, S)
        fwd = O.layer(logits, x, W1, W3, W2, k, W, S)
        ref = O.layer_backward(fwd, dout, W1, W3, W2, E)
        C = fwd["plan"]["C"]
        for name in ("dx", "dlogits"):
            got = np.concatenate([r[name] for r in ebw["ranks"]])
            assert np.allclose(got, ref[name], rtol=1e-10, atol=1e-12), name
        for u, r in enumerate(ebw["ranks"]):
            assert np.allclose(r["dy"], ref["dy"][u * C:(u + 1) * C], rtol=1e-12, atol=1e-12)
            assert np.allclose(r["dX_rows"], ref["dX_rows"][u * C:(u + 1) * C], rtol=1e-10, atol=1e-12)
        for name in ("dW1", "dW3", "dW2"):
            assert np.allclose(ebw[name], ref[name], rtol=1e-10, atol=1e-12), name
