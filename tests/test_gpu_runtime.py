"""Runtime behaviour of the layer on the GPU (needs a B200): CUDA-graph replay equals
eager execution, layers share one replica pool, and the plan kernel matches the oracle on
many random demand vectors (including slot overflow)."""
import numpy as np
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I
from oracle import moe_oracle as O

from harness import oracle_plan_fields

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()


def test_graph_replay_matches_eager():
    w = I.small_workload("g", 1000, 64, 6, 8, 8, 512, 256, alpha=0.8, seed=21)
    W = I.make_weights(w, device="cuda")
    logits, x = I.make_logits(w).cuda(), I.make_x(w).cuda()
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    eager = L.forward(logits, x, *W).clone()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g.capture_begin()
        L.forward(logits, x, *W)
        g.capture_end()
    torch.cuda.synchronize()
    L.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    assert torch.equal(L.out, eager)
    # replay on new inputs written into the captured buffers
    w2 = I.small_workload("g", 1000, 64, 6, 8, 8, 512, 256, alpha=2.0, seed=22)
    logits.copy_(I.make_logits(w2).cuda())
    x.copy_(I.make_x(w2).cuda())
    g.replay()
    torch.cuda.synchronize()
    L2 = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    ref = L2.forward(logits, x, *W)
    torch.cuda.synchronize()
    assert torch.equal(L.out, ref)
    del g


def test_layers_share_one_pool():
    """Two layers with their own weights and one replica pool, run one after the other:
    each output equals that of a layer with a private pool."""
    wa = I.small_workload("a", 512, 32, 4, 8, 4, 256, 256, alpha=2.0, seed=23)
    wb = I.small_workload("b", 512, 32, 4, 8, 4, 256, 256, alpha=1.0, seed=24)
    Wa = I.make_weights(wa, device="cuda")
    Wb = I.make_weights(I.small_workload("b", 512, 32, 4, 8, 4, 256, 256, seed=99), device="cuda")
    la, lb = I.make_logits(wa).cuda(), I.make_logits(wb).cuda()
    xa, xb = I.make_x(wa).cuda(), I.make_x(wb).cuda()
    A = M.MoELayer(512, 32, 4, 8, 4, 256, 256)
    B = M.MoELayer(512, 32, 4, 8, 4, 256, 256, pool=A.pool)
    outa = A.forward(la, xa, *Wa).clone()
    outb = B.forward(lb, xb, *Wb).clone()
    torch.cuda.synchronize()
    A2 = M.MoELayer(512, 32, 4, 8, 4, 256, 256)
    B2 = M.MoELayer(512, 32, 4, 8, 4, 256, 256)
    assert torch.equal(outa, A2.forward(la, xa, *Wa))
    assert torch.equal(outb, B2.forward(lb, xb, *Wb))
    assert int(A.err.item()) == int(B.err.item()) == 0


@pytest.mark.parametrize("E,R,S", [(8, 4, 2), (64, 8, 3), (256, 32, 4), (128, 16, 0), (96, 96, 2)])
def test_plan_random_demand(E, R, S):
    """moe_plan_balanced on random count vectors (Zipf-like and adversarial) against the
    oracle's plan: every field bit-exact, and the slot-overflow error where it occurs."""
    rng = np.random.default_rng(E * 1000 + R * 10 + S)
    L = M.plan_layout(E, R, S)
    plan = torch.empty(L.words, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    n_err = 0
    for trial in range(60):
        k = int(rng.integers(1, min(E, 8) + 1))
        T = R * int(rng.integers(1, 64))
        A = T * k
        # counts summing to A: a Zipf draw, or everything on a few experts
        if trial % 3 == 2:
            hot = rng.choice(E, size=max(1, E // 16), replace=False)
            p = np.full(E, 1e-3)
            p[hot] = 1.0
        else:
            p = (np.arange(E) + 1.0) ** -rng.uniform(0, 2.5)
        counts = rng.multinomial(A, p / p.sum()).astype(np.int32)
        ref = O.plan_balanced(counts, T, k, E, R, S)
        err.zero_()
        M.moe_plan_balanced(torch.from_numpy(counts).cuda(), T, k, R, S, plan, err)
        torch.cuda.synchronize()
        assert int(err.item()) == ref["err"], (trial, counts)
        if ref["err"]:
            n_err += 1
            continue

        class Wk:  # shape holder for oracle_plan_fields
            pass
        wk = Wk()
        wk.R, wk.S, wk.E, wk.B = R, S, E, E // R
        exp = oracle_plan_fields(ref, wk)
        sizes = dict(kept_rows=R, room_prefix=R + 1, expert_home_off=E, stream_off=E + 1,
                     replica_expert=R * S, replica_list=1 + R * S, n_groups=R,
                     groups=R * L.max_groups_per_rank * 4)
        for name, v in exp.items():
            off = getattr(L, name)
            got = plan[off:off + sizes[name]].cpu().numpy()
            assert np.array_equal(got, v), (trial, name)
    if S == 0:
        assert n_err > 0  # hot draws cannot be balanced without slots


def test_prefetch_rejects_a_corrupted_slot_list():
    """The bulk-copy prefetch checks every listed slot before copying: a slot outside
    [0, R*S) or one whose expert is outside [0, E) sets MOE_DERR_ID_RANGE and is skipped
    (nothing read or written for it); the valid slots are still copied bitwise."""
    w = I.small_workload("pf", 512, 32, 4, 8, 4, 256, 256, alpha=2.0, seed=23)
    W1, W3, W2 = I.make_weights(w, device="cuda")
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    L.route_plan(I.make_logits(w).cuda())
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    lay = M.plan_layout(w.E, w.R, w.S)
    plan = L.plan.clone()
    n = int(plan[lay.replica_list].item())
    assert n >= 2
    slots = plan[lay.replica_list + 1: lay.replica_list + 1 + n].tolist()
    good = slots[0]
    bad_expert_slot = slots[1]
    plan[lay.replica_expert + bad_expert_slot] = w.E + 3        # an expert outside [0, E)
    plan[lay.replica_list] = 3
    plan[lay.replica_list + 1] = good
    plan[lay.replica_list + 2] = bad_expert_slot
    plan[lay.replica_list + 3] = w.R * w.S + 1                   # a slot outside the pool
    P1, P3, P2 = (torch.full_like(p, 7) for p in L.pool)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_prefetch_replicas(plan, W1, W3, W2, w.R, w.S, P1, P3, P2, err)
    torch.cuda.synchronize()
    assert int(err.item()) == M.DERR_ID_RANGE
    e = int(plan[lay.replica_expert + good].item())
    assert torch.equal(P1[good], W1[e]) and torch.equal(P3[good], W3[e]) and torch.equal(P2[good], W2[e])
    for q in range(w.R * w.S):
        if q != good:
            assert bool((P1[q] == 7).all()) and bool((P2[q] == 7).all())
