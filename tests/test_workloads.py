"""The synthetic workloads hit their stated routing targets (oracle, CPU only).

Pins the input recipe: the stored bias scalars still produce the workload's maxvio (or
hot share) with the seeded logits, and the equal-load plan fits the slot budget S.
"""
import numpy as np
import pytest

from load_balanced_dispatch_warp_b200 import inputs as I
from oracle import moe_oracle as O


@pytest.mark.parametrize("name", list(I.WORKLOADS))
def test_workload_routing_targets(name):
    w = I.WORKLOADS[name]
    assert w.E % w.R == 0 and w.A % w.R == 0
    idx, gate, err = O.topk_route(I.make_logits(w).numpy(), w.k)
    assert err == 0
    h = O.expert_histogram(idx, w.E, w.R)
    assert h["err"] == 0
    if w.bias_kind == "hot":
        hot = I.hot_experts(w).numpy()
        share = h["counts"][hot].sum() / w.A
        assert abs(share - w.target) < 2e-3
    elif not np.isnan(w.target):
        assert abs(h["maxvio"] - w.target) < 5e-3 * max(1.0, w.target)
    p = O.plan_balanced(h["counts"], w.T, w.k, w.E, w.R, w.S)
    assert p["err"] == 0, "plan needs more slots than the workload's S"
    assert all(p["kept_rows"][r] + p["room_prefix"][r + 1] - p["room_prefix"][r] == w.C
               for r in range(w.R))
