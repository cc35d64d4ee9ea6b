"""The oracle's backward pins fail on plausible mistakes (CPU only).

Each case swaps one oracle function for a copy with one planted mistake (a dropped term, a
missing factor, a skipped index, a wrong derivative) and checks that the pin written for
that function fails.  The mistakes live here, in the test, never in the oracle."""
import numpy as np
import pytest

import test_oracle_backward as P
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
