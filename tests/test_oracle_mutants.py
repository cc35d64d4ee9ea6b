"""The oracle's pins fail on plausible mistakes (CPU only).

Each case swaps one oracle function for a copy with one planted mistake (ties broken the
wrong way, a softmax over the wrong set, a dropped choice, a reordered plan or placement, a
shifted row, a copied operand, swapped projections, missing gates, a dropped term, a wrong
derivative) and checks that the pin written for that function fails.  The mistakes live
here, in the test, never in the oracle."""
import json

import numpy as np
import pytest

import test_oracle_backward as P
import test_oracle_pins as F
from oracle import moe_oracle as O

ORIG = {n: getattr(O, n) for n in ("topk_backward", "combine_backward", "dispatch_backward",
                                   "expert_ffn_backward")}


def topk_backward_without_centring(gate, dgate, idx, E):
    gate = np.asarray(gate)
    T, k = idx.shape
    dl = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            dl[t, int(idx[t, j])] = gate[t, j] * dgate[t, j]  # the "- sum_i g_i dg_i" dropped
    return dl


def combine_backward_without_gate(dout, y, perm, gate):
    dy, dgate = ORIG["combine_backward"](dout, y, perm, gate)
    T, k = np.asarray(perm).shape
    for t in range(T):
        for j in range(k):
            dy[int(perm[t, j])] = np.asarray(dout[t], dtype=np.float64)  # gate factor missing
    return dy, dgate


def dispatch_backward_skipping_last_choice(dX, perm):
    dX = np.asarray(dX, dtype=np.float64)
    T, k = np.asarray(perm).shape
    dx = np.zeros((T, dX.shape[1]))
    for t in range(T):
        for j in range(k - 1):
            dx[t] += dX[int(perm[t, j])]
    return dx


def expert_ffn_backward_wrong_up_derivative(X, w1, w3, w2, dy):
    b = dict(ORIG["expert_ffn_backward"](X, w1, w3, w2, dy))
    X, w1, w3, w2, dy = (np.asarray(a, dtype=np.float64) for a in (X, w1, w3, w2, dy))
    g = X @ w1.T
    du = (dy @ w2) * O.silu_grad(g)  # silu'(g) where silu(g) belongs
    b["dw3"] = du.T @ X
    b["dX"] = b["dg"] @ w1 + du @ w3
    return b


CASES = [
    ("topk_backward", topk_backward_without_centring,
     P.test_topk_backward_matches_central_differences_of_the_gates),
    ("combine_backward", combine_backward_without_gate,
     P.test_combine_backward_is_the_adjoint_in_rows_and_in_gates),
    ("dispatch_backward", dispatch_backward_skipping_last_choice,
     P.test_dispatch_backward_is_the_adjoint_of_dispatch),
    ("expert_ffn_backward", expert_ffn_backward_wrong_up_derivative,
     P.test_expert_ffn_backward_matches_central_differences),
]


@pytest.mark.parametrize("name,mutant,pin", CASES, ids=[c[0] for c in CASES])
def test_pin_catches_planted_mistake(monkeypatch, name, mutant, pin):
    pin()  # passes on the oracle as it is
    monkeypatch.setattr(O, name, mutant)
    with pytest.raises(AssertionError):
        pin()


# ------------------------------------------------------------------ forward pieces
FWD = {n: getattr(O, n) for n in ("topk_route", "expert_histogram", "plan_balanced", "permute",
                                  "dispatch", "prefetch", "expert_ffn", "combine")}


def fixture():
    with open(F.GOLD) as f:
        g = json.load(f)
    idx = np.array([[int(p[0]), int(p[1])] for p in g["pairs"]], dtype=np.int32)
    return g, idx, np.arange(g["tokens"]) % g["ranks"]


def topk_ties_to_higher_id(logits, k):
    logits = np.asarray(logits, dtype=np.float32)
    idx, gate, err = FWD["topk_route"](logits[:, ::-1], k)
    return (logits.shape[1] - 1 - idx).astype(np.int32), gate, err


def topk_softmax_over_all_experts(logits, k):
    idx, gate, err = FWD["topk_route"](logits, k)
    row = np.asarray(logits, dtype=np.float64)
    ex = np.exp(row - row.max(axis=1, keepdims=True))
    full = ex / ex.sum(axis=1, keepdims=True)
    return idx, np.take_along_axis(full, idx.astype(np.int64), axis=1), err


def histogram_of_first_choice(idx, E, R, expert_to_rank=None):
    idx = np.asarray(idx)
    return FWD["expert_histogram"](idx[:, :1], E, R, expert_to_rank)


def histogram_without_mapping_check(idx, E, R, expert_to_rank=None):
    """The rank sum with Python indexing and no range check: -1 wraps to rank R-1, R is
    clipped to rank R-1, and no error bit is set."""
    h = FWD["expert_histogram"](idx, E, R)
    m = O.home_rank_map(E, R) if expert_to_rank is None else np.asarray(expert_to_rank)
    loads = np.zeros(R, dtype=np.int64)
    for e in range(E):
        loads[min(int(m[e]), R - 1)] += h["counts"][e]
    h["loads"] = loads
    h["err"] = O.validate_trace(idx, E)
    return h


def plan_groups_reversed(counts, T, k, E, R, S):
    p = FWD["plan_balanced"](counts, T, k, E, R, S)
    p["groups"] = [list(reversed(g)) for g in p["groups"]]
    return p


def permute_unstable(idx, plan, E, R):
    perm, src = FWD["permute"](idx, plan, E, R)
    perm, src = np.array(perm), np.array(src)
    e = int(np.asarray(idx)[0, 0])  # the rows of one expert, in reverse token order
    where = [(t, j) for t in range(len(idx)) for j in range(len(idx[0])) if idx[t][j] == e]
    rows = [perm[t, j] for t, j in where][::-1]
    for (t, j), r in zip(where, rows):
        perm[t, j] = r
        src[r] = t
    return perm, src


def dispatch_shifted(x, src):
    return np.asarray(x)[np.roll(np.asarray(src), 1)]


def prefetch_w1_twice(plan, W1, W3, W2, R, S):
    return {s: (a, a, c) for s, (a, b, c) in FWD["prefetch"](plan, W1, W3, W2, R, S).items()}


def ffn_gate_and_up_swapped(X, w1, w3, w2):
    return FWD["expert_ffn"](X, w3, w1, w2)


def combine_without_gates(y, perm, gate, tokens=None):
    return FWD["combine"](y, perm, np.ones_like(np.asarray(gate, dtype=np.float64)), tokens)


FWD_CASES = [
    ("topk_route", topk_ties_to_higher_id, F.test_topk_bruteforce_with_ties),
    ("topk_route", topk_softmax_over_all_experts, F.test_topk_special_cases),
    ("expert_histogram", histogram_of_first_choice,
     lambda: F.test_fixture_demand_and_balancedness(fixture())),
    ("expert_histogram", histogram_without_mapping_check,
     lambda: F.test_fixture_mapping_must_cover_every_expert(fixture())),
    ("plan_balanced", plan_groups_reversed, lambda: F.test_fixture_plan_derived_by_hand(fixture())),
    ("permute", permute_unstable, lambda: F.test_fixture_plan_derived_by_hand(fixture())),
    ("dispatch", dispatch_shifted, F.test_dispatch_prefetch_identities),
    ("prefetch", prefetch_w1_twice, F.test_dispatch_prefetch_identities),
    ("expert_ffn", ffn_gate_and_up_swapped, F.test_ffn_closed_forms),
    ("combine", combine_without_gates, F.test_combine_identity_and_scaled_experts),
]


@pytest.mark.parametrize("name,mutant,pin", FWD_CASES,
                         ids=[f"{c[0]}-{c[1].__name__}" for c in FWD_CASES])
def test_forward_pin_catches_planted_mistake(monkeypatch, name, mutant, pin):
    pin()
    monkeypatch.setattr(O, name, mutant)
    with pytest.raises(AssertionError):
        pin()


# ------------------------------------------------------------------ ledgers and variants
VAR = {n: getattr(O, n) for n in ("validate_trace", "capacity_ledger", "remote_routes",
                                  "topk_route_biased", "dispatch_capacity", "combine")}


def capacity_keeps_the_last_assignments(idx, E, cap):
    """Keeps the LAST cap assignments of each expert (reverse token order)."""
    idx = np.asarray(idx)
    T = idx.shape[0]
    perm, src, rows = VAR["dispatch_capacity"](idx[::-1], E, cap)
    perm = perm[::-1].copy()
    src = np.where(src >= 0, T - 1 - src, -1).astype(np.int32)
    return perm, src, rows


def capacity_padding_absorbs_overflow(idx, E, cap):
    """Padding computed as cap - demand, so overflow cancels padding in the totals."""
    perm, src, rows = VAR["dispatch_capacity"](idx, E, cap)
    rows = dict(rows)
    rows["padding"] = cap - (rows["processed"] + rows["overflow"])
    return perm, src, rows


def combine_reads_dropped_rows(y, perm, gate, tokens=None):
    """A dropped assignment (perm = -1) read as the last row of y instead of left out."""
    perm = np.asarray(perm)
    y = np.asarray(y)
    return VAR["combine"](y, np.where(perm < 0, len(y) - 1, perm), gate, tokens)


def validate_without_repeat_check(idx, E):
    return VAR["validate_trace"](idx, E) & ~O.ERR_DUPLICATE


def ledger_overflow_unclamped(counts, A, E, cf_num=5, cf_den=4):
    led = VAR["capacity_ledger"](counts, A, E, cf_num, cf_den)
    led["overflow"] = np.asarray(counts, dtype=np.int64) - led["cap"]
    return led


def remote_counts_local_routes(idx, origin, expert_to_rank):
    return np.asarray(idx).size - VAR["remote_routes"](idx, origin, expert_to_rank)


def biased_gate_from_biased_scores(logits, bias, k):
    idx, _, err = VAR["topk_route_biased"](logits, bias, k)
    sc = np.asarray(logits, dtype=np.float64) + np.asarray(bias, dtype=np.float64)
    sel = np.take_along_axis(sc, idx.astype(np.int64), axis=1)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    return idx, ex / ex.sum(axis=1, keepdims=True), err


VAR_CASES = [
    ("validate_trace", validate_without_repeat_check,
     lambda: F.test_fixture_validation_rules(fixture())),
    ("capacity_ledger", ledger_overflow_unclamped, lambda: F.test_fixture_capacity_ledger(fixture())),
    ("remote_routes", remote_counts_local_routes, lambda: F.test_fixture_remote_routes(fixture())),
    ("topk_route_biased", biased_gate_from_biased_scores, F.test_biased_topk_pins),
    ("dispatch_capacity", capacity_keeps_the_last_assignments,
     lambda: F.test_fixture_fixed_capacity_dispatch(fixture())),
    ("dispatch_capacity", capacity_padding_absorbs_overflow,
     lambda: F.test_fixture_fixed_capacity_dispatch(fixture())),
    ("combine", combine_reads_dropped_rows, F.test_combine_leaves_dropped_assignments_out),
]


@pytest.mark.parametrize("name,mutant,pin", VAR_CASES,
                         ids=[f"{c[0]}-{c[1].__name__}" for c in VAR_CASES])
def test_ledger_and_variant_pins_catch_planted_mistakes(monkeypatch, name, mutant, pin):
    pin()
    monkeypatch.setattr(O, name, mutant)
    with pytest.raises(AssertionError):
        pin()


# ------------------------------------------------------------------ expert parallelism
EPF = {n: getattr(O, n) for n in ("ep_rank_base", "ep_permute")}


def rank_base_including_own_rank(counts_all, me):
    """Counts rank me's own assignments into its base as well."""
    return np.asarray(counts_all, dtype=np.int64)[:me + 1].sum(axis=0)


def ep_permute_local_order_only(idx_local, q_base, plan, E, R):
    """Ranks each assignment within its own rank's tokens only (base dropped)."""
    return EPF["ep_permute"](idx_local, np.zeros_like(np.asarray(q_base)), plan, E, R)


EP_MUTANTS = [
    ("ep_rank_base", rank_base_including_own_rank,
     F.test_ep_rank_base_counts_the_lower_ranks_assignments),
    ("ep_rank_base", rank_base_including_own_rank,
     F.test_ep_layer_is_the_layer_of_the_rank_major_batch),
    ("ep_permute", ep_permute_local_order_only,
     F.test_ep_layer_is_the_layer_of_the_rank_major_batch),
]


@pytest.mark.parametrize("name,mutant,pin", EP_MUTANTS,
                         ids=[f"{c[0]}-{c[1].__name__}-{c[2].__name__}" for c in EP_MUTANTS])
def test_ep_pins_catch_planted_mistakes(monkeypatch, name, mutant, pin):
    pin()
    monkeypatch.setattr(O, name, mutant)
    # a base that overshoots can push a stream position past the last rank's room, where
    # the placement rule finds no rank: that is caught too
    with pytest.raises((AssertionError, IndexError)):
        pin()


def ep_backward_keeping_replicas_away(ep, douts, W1, W3, W2, E, S):
    """Replica gradients left on the ranks that computed them (no reduction back home)."""
    plan = dict(ep["plan"])
    plan["replica_expert"] = [-1] * len(plan["replica_expert"])
    return EPB["ep_layer_backward"](dict(ep, plan=plan), douts, W1, W3, W2, E, S)


EPB = {"ep_layer_backward": O.ep_layer_backward}


@pytest.mark.parametrize("mutant", [ep_backward_keeping_replicas_away])
def test_ep_backward_pin_catches_planted_mistake(monkeypatch, mutant):
    F.test_ep_backward_is_the_backward_of_the_rank_major_batch()
    monkeypatch.setattr(O, "ep_layer_backward", mutant)
    with pytest.raises(AssertionError):
        F.test_ep_backward_is_the_backward_of_the_rank_major_batch()
