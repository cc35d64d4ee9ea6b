"""Bisect the scalar of each workload's logit-bias recipe against the oracle.

Writes ``load_balanced_dispatch_warp_b200/workload_bias.json``: for every workload whose
recipe scalar is not fixed, the scalar (alpha, sigma or beta) at which the oracle's
rank-level maxvio (or, for the hotspot recipe, the share of assignments taken by the
hot experts) reaches the workload's target.  Calls only the oracle and the seeded input
generators.  Usage:  python oracle/calibrate_workloads.py [name ...]
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from oracle import moe_oracle as O  # noqa: E402
from load_balanced_dispatch_warp_b200 import inputs as I  # noqa: E402


def measure(w, param):
    logits = I.make_logits(w, param).numpy()
    idx, _, err = O.topk_route(logits, w.k)
    assert err == 0
    h = O.expert_histogram(idx, w.E, w.R)
    if w.bias_kind == "hot":
        hot = set(int(e) for e in I.hot_experts(w))
        share = sum(int(h["counts"][e]) for e in hot) / w.A
        return share, h["maxvio"]
    return h["maxvio"], h["maxvio"]


def bisect(w, lo, hi, iters=30):
    f_lo = measure(w, lo)[0]
    f_hi = measure(w, hi)[0]
    while f_hi < w.target:
        lo, f_lo = hi, f_hi
        hi *= 2.0
        f_hi = measure(w, hi)[0]
    best = (abs(f_hi - w.target), hi)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        f = measure(w, mid)[0]
        best = min(best, (abs(f - w.target), mid))
        if f < w.target:
            lo = mid
        else:
            hi = mid
        if abs(f - w.target) <= 1e-3 * max(1.0, w.target):
            break
    return best[1]


def main(names):
    out = I.load_bias_params()
    for name in names:
        w = I.WORKLOADS[name]
        if w.fixed_param is not None:
            continue
        p = bisect(w, 0.0, 1.0)
        val, mv = measure(w, p)
        out[name] = dict(param=p, recipe=w.bias_kind, target=w.target, achieved=val, maxvio=mv)
        print(name, out[name], flush=True)
    with open(I.BIAS_FILE, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:] or [n for n, w in I.WORKLOADS.items() if w.fixed_param is None])
