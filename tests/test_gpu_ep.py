"""Expert parallelism across GPUs on one B200.

W ranks run inside one process (``LocalRanks``): each rank's buffers are separate
allocations, addressed by its peers through the pointer tables, and the stages run rank by
rank in the order the barriers give across processes.  Checked against the oracle's
W-process layer (bit-exact integers and rows, the FFN tolerance on y and out) and, bit for
bit, against the single-GPU layer of the concatenated batch with R = W at full workload
sizes.  A last case runs two real processes on the one GPU, each rank mapping the other's
buffers through CUDA IPC, with the exchange over gloo."""
import os
import socket

import numpy as np
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from harness import assert_close_scaled, make_inputs, oracle_plan_fields, to64
from load_balanced_dispatch_warp_b200 import inputs as I
from load_balanced_dispatch_warp_b200.ep import EPRank, LocalRanks
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def make_ranks(w, weights):
    W1, W3, W2 = weights
    W, B, T = w.R, w.E // w.R, w.T // w.R
    return LocalRanks([EPRank(u, W, T, w.E, w.k, w.S, W1[u * B:(u + 1) * B],
                              W3[u * B:(u + 1) * B], W2[u * B:(u + 1) * B]) for u in range(W)])


def shards(t, W):
    T = t.shape[0] // W
    return [t[u * T:(u + 1) * T].contiguous() for u in range(W)]


def plan_fields(plan, E, W, S):
    """The plan's fields (the words between them are padding, left as allocated)."""
    L = M.plan_layout(E, W, S)
    sizes = dict(kept_rows=W, room_prefix=W + 1, expert_home_off=E, stream_off=E + 1,
                 replica_expert=W * S, replica_list=1 + W * S, n_groups=W,
                 groups=W * L.max_groups_per_rank * 4)
    return {n: plan[getattr(L, n):getattr(L, n) + sz].cpu().numpy() for n, sz in sizes.items()}


# (name, T, E, k, W, S, d, F): W = 1 (the single-GPU layer), a ragged last tile, top-3,
# several tiles per rank, 8 ranks of 8 experts, 64 ranks, no pool slots
SMALL = [("ep_w1", 64, 8, 2, 1, 2, 128, 256), ("ep_w2", 96, 8, 2, 2, 4, 128, 256),
         ("ep_w4", 256, 16, 4, 4, 4, 256, 128), ("ep_w4_k3", 200, 32, 3, 4, 6, 128, 384),
         ("ep_w8", 512, 64, 6, 8, 8, 256, 256), ("ep_w2_tiles", 1200, 8, 2, 2, 3, 128, 128),
         # the most ranks a table holds (64), 4 tokens each; no pool slots (a skewed trace
         # then needs copies it cannot place: MOE_DERR_SLOTS on every rank)
         ("ep_w64", 256, 128, 2, 64, 2, 128, 128), ("ep_w4_nopool", 128, 16, 2, 4, 0, 128, 128)]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_ep_ranks_match_the_oracle(case):
    w = I.small_workload(*case, alpha=1.2)
    W = w.R
    logits, x, weights = make_inputs(w)
    lr = make_ranks(w, weights)
    lr.forward([s.cuda() for s in shards(logits, W)], [s.cuda() for s in shards(x, W)])
    torch.cuda.synchronize()
    w64 = tuple(to64(t) for t in weights)
    ref = O.ep_layer(np.split(logits.numpy(), W), np.split(to64(x), W), *w64, w.k, w.S)
    if ref["err"]:  # e.g. a plan that needs slots when there are none: every rank flags it
        for r in lr.ranks:
            assert int(r.err.item()) == ref["err"]
        return
    idx_all = np.concatenate([rr["idx"] for rr in ref["ranks"]])
    hist = O.expert_histogram(idx_all, w.E, W)
    expect_plan = oracle_plan_fields(ref["plan"], w)
    for u, r in enumerate(lr.ranks):
        rr = ref["ranks"][u]
        assert int(r.err.item()) == 0
        assert np.array_equal(r.idx.cpu().numpy(), rr["idx"])
        assert np.abs(r.gate.cpu().double().numpy() - rr["gate"]).max() <= 1e-6
        assert np.array_equal(r.send.cpu().numpy(), np.append(ref["counts_all"][u], 0))
        assert np.array_equal(r.counts.cpu().numpy(), ref["counts_all"].sum(axis=0))
        assert np.array_equal(r.q_base.cpu().numpy(), O.ep_rank_base(ref["counts_all"], u))
        assert np.array_equal(r.loads.cpu().numpy(), hist["loads"])
        assert r.maxvio.item() == hist["maxvio"] and r.balancedness.item() == hist["balancedness"]
        got = plan_fields(r.plan, w.E, W, w.S)
        for name, v in expect_plan.items():
            assert np.array_equal(got[name], v), f"rank {u} plan field {name}"
        assert np.array_equal(r.perm.cpu().numpy(), rr["perm"]), f"rank {u} perm"
        assert np.array_equal(to64(r.recv), rr["recv"]), f"rank {u} receive rows"
        for s in range(w.S):
            e = ref["plan"]["replica_expert"][u * w.S + s]
            if e >= 0:
                assert torch.equal(r.P1[s], weights[0][e]) and torch.equal(r.P3[s], weights[1][e])
                assert torch.equal(r.P2[s], weights[2][e])
        assert_close_scaled(to64(r.y), rr["y"], f"rank {u} y")
        assert_close_scaled(to64(r.out), rr["out"], f"rank {u} out")


FULL = ["near_balanced", "qwen_mv1", "mixtral", "deepseek"]


@pytest.mark.parametrize("name", FULL)
def test_ep_is_the_single_gpu_layer_bit_for_bit(name):
    """W = R ranks on the workload's shards against MoELayer on the whole batch: the same
    plan, rows, y and out, bit for bit."""
    w = I.WORKLOADS[name]
    W = w.R
    logits, x, weights = make_inputs(w)
    lg, xd = logits.cuda(), x.cuda()
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    L.forward(lg, xd, *weights)
    lr = make_ranks(w, weights)
    lr.forward(shards(lg, W), shards(xd, W))
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    C = w.C
    for u, r in enumerate(lr.ranks):
        assert int(r.err.item()) == 0
        ref_plan = plan_fields(L.plan, w.E, W, w.S)
        for fname, v in plan_fields(r.plan, w.E, W, w.S).items():
            assert np.array_equal(v, ref_plan[fname]), f"rank {u} plan field {fname}"
        assert torch.equal(r.counts, L.counts) and torch.equal(r.loads, L.loads)
        assert r.maxvio.item() == L.maxvio.item()
        assert torch.equal(r.perm, L.perm[u * r.T:(u + 1) * r.T]), f"rank {u} perm"
        assert torch.equal(r.recv, L.recv[u * C:(u + 1) * C]), f"rank {u} receive rows"
        assert torch.equal(r.y, L.y[u * C:(u + 1) * C]), f"rank {u} y"
        assert torch.equal(r.out, L.out[u * r.T:(u + 1) * r.T]), f"rank {u} out"


def test_ep_error_on_one_rank_stops_every_rank():
    """A non-finite logit on rank 1 reaches every rank through the exchanged vectors."""
    w = I.small_workload("ep_err", 64, 8, 2, 2, 2, 128, 128)
    logits, x, weights = make_inputs(w)
    logits[40, 3] = float("nan")
    lr = make_ranks(w, weights)
    lr.forward([s.cuda() for s in shards(logits, 2)], [s.cuda() for s in shards(x, 2)])
    torch.cuda.synchronize()
    for r in lr.ranks:
        assert int(r.err.item()) & M.DERR_NONFINITE
    assert int(lr.ranks[1].send[-1].item()) & M.DERR_NONFINITE
    assert int(lr.ranks[0].send[-1].item()) == 0


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


IPC_CASE = ("ep_ipc", 256, 16, 4, 2, 4, 256, 256)


def _ipc_worker(rank, world, port, path):
    import torch.distributed as dist
    from load_balanced_dispatch_warp_b200.ep import EPLayer, GlooComm
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        w = I.small_workload(*IPC_CASE, alpha=1.2)
        logits, x, weights = make_inputs(w)
        B, T = w.E // world, w.T // world
        own = tuple(t[rank * B:(rank + 1) * B].contiguous() for t in weights)
        layer = EPLayer(GlooComm(), T, w.E, w.k, w.S, *own)
        out = layer.forward(shards(logits, world)[rank].cuda(), shards(x, world)[rank].cuda())
        torch.cuda.synchronize()
        torch.save({"out": out.cpu(), "err": int(layer.rank.err.item()),
                    "perm": layer.rank.perm.cpu()}, f"{path}.{rank}")
        dist.barrier()  # no rank unmaps or frees while a peer may still read its buffers
        layer.close()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ep_two_processes_through_ipc(tmp_path):
    """Two processes on the one GPU, each a rank holding its own buffers, its peer's
    receive buffer, y and weights mapped through CUDA IPC: the result equals the one-process
    ranks bit for bit."""
    import torch.multiprocessing as mp
    if not _gpu_compute_mode_default():
        pytest.skip("two processes on one GPU need the Default compute mode")
    world = 2
    path = str(tmp_path / "ep_out")
    mp.spawn(_ipc_worker, args=(world, _free_port(), path), nprocs=world, join=True)
    w = I.small_workload(*IPC_CASE, alpha=1.2)
    logits, x, weights = make_inputs(w)
    lr = make_ranks(w, weights)
    lr.forward([s.cuda() for s in shards(logits, world)], [s.cuda() for s in shards(x, world)])
    torch.cuda.synchronize()
    for u in range(world):
        got = torch.load(f"{path}.{u}")
        assert got["err"] == 0
        assert torch.equal(got["perm"], lr.ranks[u].perm.cpu())
        assert torch.equal(got["out"], lr.ranks[u].out.cpu()), f"rank {u} out"


def _gpu_compute_mode_default():
    import subprocess
    try:
        out = subprocess.run(["nvidia-smi", "--query-gpu=compute_mode", "--format=csv,noheader",
                              "-i", "0"], capture_output=True, text=True, timeout=30).stdout
    except (OSError, subprocess.SubprocessError):
        return False
    return out.strip() == "Default"


def _nccl_worker(rank, world, port, path):
    import torch.distributed as dist
    from load_balanced_dispatch_warp_b200.ep import EPLayer, NcclComm
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=rank, world_size=world,
                            device_id=torch.device("cuda", 0))
    try:
        w = I.small_workload(*IPC_CASE[:4], 1, *IPC_CASE[5:], alpha=1.2)
        logits, x, weights = make_inputs(w)
        layer = EPLayer(NcclComm(), w.T, w.E, w.k, w.S, *weights)
        for _ in range(2):  # a second step reuses every buffer
            out = layer.forward(logits.cuda(), x.cuda())
        torch.cuda.synchronize()
        torch.save({"out": out.cpu(), "err": int(layer.rank.err.item())}, path)
        layer.close()
    finally:
        dist.destroy_process_group()


def test_ep_nccl_communicator_single_rank(tmp_path):
    """The NCCL communicator's all-gather and barriers on a one-rank group: the layer's
    output equals the single-GPU layer's, bit for bit."""
    import torch.multiprocessing as mp
    path = str(tmp_path / "ep_nccl")
    mp.spawn(_nccl_worker, args=(1, _free_port(), path), nprocs=1, join=True)
    w = I.small_workload(*IPC_CASE[:4], 1, *IPC_CASE[5:], alpha=1.2)
    logits, x, weights = make_inputs(w)
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    L.forward(logits.cuda(), x.cuda(), *weights)
    torch.cuda.synchronize()
    got = torch.load(path)
    assert got["err"] == 0
    assert torch.equal(got["out"], L.out.cpu())


# ------------------------------------------------------------------------------ backward
BWD_SMALL = [("epb_w2", 96, 8, 2, 2, 4, 128, 256), ("epb_w4_k3", 200, 32, 3, 4, 6, 128, 384),
             ("epb_w8", 512, 64, 6, 8, 8, 256, 256), ("epb_hot", 512, 32, 4, 8, 4, 128, 256)]
BWD_FULL = ["near_balanced", "qwen_mv1", "mixtral"]


def _ep_backward_against_layer(w, alpha=None):
    W = w.R
    logits, x, weights = make_inputs(w)
    g = torch.Generator().manual_seed(41)
    dout = torch.randn(w.T, w.d, generator=g).to(torch.bfloat16).cuda()
    lg, xd = logits.cuda(), x.cuda()
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    L.forward(lg, xd, *weights)
    b = L.backward(dout, *weights)
    lr = make_ranks(w, weights)
    lr.forward(shards(lg, W), shards(xd, W))
    lr.backward(shards(dout, W))
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    C, Tl = w.C, w.T // W
    for u, r in enumerate(lr.ranks):
        assert int(r.err.item()) == 0
        assert torch.equal(r.dy, b["dy"][u * C:(u + 1) * C]), f"rank {u} dy"
        assert torch.equal(r.dgate, b["dgate"][u * Tl:(u + 1) * Tl]), f"rank {u} dgate"
        assert torch.equal(r.dx_rows, b["dx_rows"][u * C:(u + 1) * C]), f"rank {u} dx rows"
        assert torch.equal(r.dx, b["dx"][u * Tl:(u + 1) * Tl]), f"rank {u} dx"
        assert torch.equal(r.dlogits, b["dlogits"][u * Tl:(u + 1) * Tl]), f"rank {u} dlogits"
    # the same fp32 sums of the same products, associated differently (a home expert's own
    # groups, then each copy's partial): a missing or doubled copy would be off by O(1)
    for name in ("dW1", "dW3", "dW2"):
        ep = torch.cat([getattr(r, name) for r in lr.ranks])
        ref = b[name]
        tol = 1e-4 * ref.abs().amax(dim=(1, 2), keepdim=True) + 1e-6
        bad = (ep - ref).abs() > tol
        assert not bad.any(), f"{name}: {int(bad.sum())} entries off"
    n_rep = int(lr.ranks[0].plan[M.plan_layout(w.E, W, w.S).replica_list].item())
    return n_rep


@pytest.mark.parametrize("case", BWD_SMALL, ids=[c[0] for c in BWD_SMALL])
def test_ep_backward_is_the_single_gpu_backward(case):
    w = I.small_workload(*case, alpha=1.2 if case[0] != "epb_hot" else 2.5)
    n_rep = _ep_backward_against_layer(w)
    if case[0] == "epb_hot":
        assert n_rep >= 1  # replica gradients crossed ranks


@pytest.mark.parametrize("name", BWD_FULL)
def test_ep_backward_full_size(name):
    n_rep = _ep_backward_against_layer(I.WORKLOADS[name])
    assert n_rep >= 1
    torch.cuda.empty_cache()


def test_ep_ranks_without_tokens():
    """T = 0 on every rank: every call returns at once, nothing is flagged."""
    w = I.small_workload("ep_empty_ref", 16, 8, 2, 2, 2, 128, 128)
    _, _, weights = make_inputs(w)
    W1, W3, W2 = weights
    lr = LocalRanks([EPRank(u, 2, 0, 8, 2, 2, W1[u * 4:(u + 1) * 4], W3[u * 4:(u + 1) * 4],
                            W2[u * 4:(u + 1) * 4]) for u in range(2)])
    empty_l = torch.zeros(0, 8, dtype=torch.float32, device="cuda")
    empty_x = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    outs = lr.forward([empty_l, empty_l], [empty_x, empty_x])
    torch.cuda.synchronize()
    for r, o in zip(lr.ranks, outs):
        assert int(r.err.item()) == 0 and o.shape == (0, 128)
        assert int(r.counts.sum().item()) == 0
