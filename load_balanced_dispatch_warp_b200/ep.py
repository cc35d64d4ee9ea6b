"""Expert parallelism across GPUs: the MoE layer with one process per GPU.

Rank ``me`` of ``W`` holds its own ``T`` tokens, the home experts [me*B, (me+1)*B) of the
E experts (B = E/W), ``S`` pool slots for redundant copies and one static receive buffer of
C = T*k rows.  A step (the MoonEP news article, paragraphs 2-3; "DeepEP-on-EFA Guidance,
section 1: What is MoE", phases (a)-(d)):

  1. route its tokens (moe_topk) and pack its demand and error word (moe_ep_counts);
  2. all-gather those vectors, so every rank computes the same plan of the whole job, its
     base offsets in every expert's token order, and the job's maxvio (moe_ep_plan);
  3. pull the weights of its planned replicas from their home ranks (moe_ep_prefetch);
  4. store every assignment's token row straight into its final row on the rank the plan
     gives it (moe_ep_dispatch, peer stores);  -- barrier --
  5. run the grouped FFN on its own C rows (moe_ep_grouped_ffn);  -- barrier --
  6. gather every one of its tokens' k rows back from the ranks that processed them, with
     the gate-weighted sum (moe_ep_combine, peer loads).
The job's token order is rank-major, so the job computes exactly the single-GPU layer of
the concatenated batch with R = W ranks (the same plan, rows and sums).

Every step runs in the library's kernels; this module only owns buffers and orders the
calls.  The all-gather and the barriers come from a communicator:
  - ``NcclComm``: torch.distributed with NCCL (one process per GPU), stream-ordered; the
    pointer tables through CUDA IPC;
  - ``GlooComm``: any torch.distributed group (e.g. gloo), synchronising the host at every
    exchange -- for processes that cannot use NCCL, such as several ranks sharing one GPU;
  - ``LocalRanks``: W ranks inside one process on one GPU (each rank's buffers are
    separate allocations; the stages run rank by rank, every rank's dispatch before any
    rank's FFN, which is the order the barriers give across processes).
"""
from __future__ import annotations

import torch

from . import (dispatch_workspace_words, ep_ffn_backward_workspace_bytes, ipc_close, ipc_export,
               ipc_import, moe_ep_combine, moe_ep_combine_backward, moe_ep_counts,
               moe_ep_dispatch, moe_ep_dispatch_backward, moe_ep_grouped_ffn,
               moe_ep_grouped_ffn_backward, moe_ep_plan, moe_ep_prefetch, moe_ep_reduce_home,
               moe_topk, moe_topk_backward, plan_layout)

SHARED = ("recv", "y", "W1", "W3", "W2")  # the buffers every rank addresses on its peers
SHARED_BWD = ("dy", "dx_rows", "dP1", "dP3", "dP2")  # and those of the backward


class EPRank:
    """Buffers and per-step calls of rank ``me`` of ``W``.

    W1, W3 [B,F,d] bf16 and W2 [B,d,F] fp16 are this rank's home experts, on its GPU.
    ``tables`` (set by the communicator) maps each name in SHARED to the W device
    pointers of that buffer on every rank, as addressed from this process."""

    def __init__(self, me: int, W: int, T: int, E: int, k: int, S: int, W1, W3, W2):
        B, F, d = W1.shape
        if B * W != E:
            raise ValueError(f"rank holds {B} experts, expected E/W = {E}/{W}")
        self.me, self.W, self.T, self.E, self.k, self.S = me, W, T, E, k, S
        self.B, self.F, self.d, self.C = B, F, d, T * k
        dev = W1.device
        i32 = dict(dtype=torch.int32, device=dev)
        self.W1, self.W3, self.W2 = W1, W3, W2
        self.idx = torch.zeros(T, k, **i32)
        self.gate = torch.zeros(T, k, dtype=torch.float32, device=dev)
        self.err = torch.zeros(1, **i32)
        self.send = torch.zeros(E + 1, **i32)
        self.gathered = torch.zeros(W, E + 1, **i32)
        self.counts = torch.zeros(E, **i32)
        self.q_base = torch.zeros(E, **i32)
        self.loads = torch.zeros(W, **i32)
        self.maxvio = torch.zeros(1, dtype=torch.float64, device=dev)
        self.balancedness = torch.zeros(1, dtype=torch.float64, device=dev)
        self.plan = torch.zeros(plan_layout(E, W, S).words, **i32)
        self.ws = torch.zeros(max(1, dispatch_workspace_words(T, E)), **i32)
        self.perm = torch.zeros(T, k, **i32)
        self.recv = torch.zeros(self.C, d, dtype=torch.bfloat16, device=dev)
        self.h = torch.zeros(self.C, F, dtype=torch.float16, device=dev)
        self.y = torch.zeros(self.C, d, dtype=torch.bfloat16, device=dev)
        self.out = torch.zeros(T, d, dtype=torch.bfloat16, device=dev)
        ns = max(S, 1)
        self.P1 = torch.zeros(ns, F, d, dtype=torch.bfloat16, device=dev)
        self.P3 = torch.zeros(ns, F, d, dtype=torch.bfloat16, device=dev)
        self.P2 = torch.zeros(ns, d, F, dtype=torch.float16, device=dev)
        self.groups_ws = torch.zeros(4 * (B + S), **i32)
        self.tables = None

    def shared(self) -> dict:
        return {"recv": self.recv, "y": self.y, "W1": self.W1, "W3": self.W3, "W2": self.W2}

    def alloc_backward(self):
        """Buffers of the backward: dy and dx rows [C,d], the weight-gradient partials of
        its groups [B+S,...] (home experts, then pool slots; the first B entries become the
        home experts' gradients), dx [T,d], dlogits [T,E]."""
        if hasattr(self, "dy"):
            return
        dev = self.W1.device
        f32, bf = torch.float32, torch.bfloat16
        B, S, F, d, C, T = self.B, self.S, self.F, self.d, self.C, self.T
        self.dy = torch.zeros(C, d, dtype=bf, device=dev)
        self.dgate = torch.zeros(T, self.k, dtype=f32, device=dev)
        self.dx_rows = torch.zeros(C, d, dtype=bf, device=dev)
        self.dP1 = torch.zeros(B + S, F, d, dtype=f32, device=dev)
        self.dP3 = torch.zeros(B + S, F, d, dtype=f32, device=dev)
        self.dP2 = torch.zeros(B + S, d, F, dtype=f32, device=dev)
        # the home experts' gradients: entries 0..B-1 of the partials, completed in place
        self.dW1, self.dW3, self.dW2 = self.dP1[:B], self.dP3[:B], self.dP2[:B]
        self.dx = torch.zeros(T, d, dtype=bf, device=dev)
        self.dlogits = torch.zeros(T, self.E, dtype=f32, device=dev)
        ws = ep_ffn_backward_workspace_bytes(T, self.k, self.E, self.W, S, d, F)
        self.bwd_ws = torch.zeros(max(ws, 256), dtype=torch.uint8, device=dev)

    def shared_backward(self) -> dict:
        self.alloc_backward()
        return {"dy": self.dy, "dx_rows": self.dx_rows, "dP1": self.dP1, "dP3": self.dP3,
                "dP2": self.dP2}

    # ---- the steps, in order
    def route(self, logits):
        moe_topk(logits, self.k, self.idx, self.gate, self.err)
        moe_ep_counts(self.idx, self.E, self.err, self.send)

    def plan_step(self):
        moe_ep_plan(self.gathered, self.me, self.T, self.k, self.S, self.counts, self.q_base,
                    self.loads, self.maxvio, self.balancedness, self.plan, self.err)

    def prefetch(self):
        t = self.tables
        moe_ep_prefetch(self.plan, t["W1"], t["W3"], t["W2"], self.me, self.E, self.S, self.d,
                        self.F, self.P1, self.P3, self.P2, self.err)

    def dispatch(self, x):
        moe_ep_dispatch(x, self.idx, self.q_base, self.plan, self.E, self.S, self.ws,
                        self.tables["recv"], self.perm, self.err)

    def ffn(self):
        moe_ep_grouped_ffn(self.recv, self.plan, self.W, self.me, self.W1, self.W3, self.W2,
                           self.P1, self.P3, self.P2, self.T, self.k, self.E, self.S,
                           self.groups_ws, self.h, self.y, self.err)

    def combine(self):
        moe_ep_combine(self.tables["y"], self.perm, self.gate, self.d, self.out, self.err)

    # ---- the backward steps, in order (the tables must hold SHARED_BWD too)
    def bwd_combine(self, dout):
        moe_ep_combine_backward(dout, self.tables["y"], self.perm, self.gate, self.tables["dy"],
                                self.dgate, self.err)

    def bwd_ffn(self):
        moe_ep_grouped_ffn_backward(self.recv, self.dy, self.plan, self.W, self.me, self.W1,
                                    self.W3, self.W2, self.P1, self.P3, self.P2, self.T, self.k,
                                    self.E, self.S, self.groups_ws, self.dx_rows, self.dP1,
                                    self.dP3, self.dP2, self.bwd_ws, self.err)

    def bwd_reduce(self):
        t = self.tables
        moe_ep_reduce_home(self.plan, t["dP1"], t["dP3"], t["dP2"], self.me, self.E, self.S,
                           self.d, self.F, self.err)

    def bwd_dispatch(self):
        moe_ep_dispatch_backward(self.tables["dx_rows"], self.perm, self.d, self.dx, self.err)

    def bwd_gates(self):
        moe_topk_backward(self.gate, self.dgate, self.idx, self.E, self.dlogits, self.err)

    def grads(self) -> dict:
        return {"dx": self.dx, "dlogits": self.dlogits, "dW1": self.dW1, "dW3": self.dW3,
                "dW2": self.dW2}


def exchange_pointers(local: dict, me: int, W: int, gather_objects, export, import_base):
    """Pointer tables of the buffers in ``local`` ({name: tensor}) on every rank.

    Each rank exports (handle, offset) for each of its buffers; ``gather_objects(obj)``
    returns every rank's object in rank order (all_gather_object); a peer's allocation is
    mapped once (``import_base(handle)`` -> base address) however many of its buffers it
    holds.  Returns ({name: [W pointers]}, [mapped bases, to close])."""
    mine = {name: export(t) for name, t in local.items()}
    everyone = gather_objects(mine)
    if len(everyone) != W:
        raise RuntimeError(f"pointer exchange: {len(everyone)} ranks answered, expected {W}")
    mapped = {}
    tables = {}
    for name, t in local.items():
        row = []
        for u in range(W):
            if u == me:
                row.append(int(t.data_ptr()))
                continue
            handle, offset = everyone[u][name]
            key = (u, bytes(handle))
            if key not in mapped:
                mapped[key] = import_base(handle)
            row.append(mapped[key] + int(offset))
        tables[name] = row
    return tables, list(mapped.values())


def _import_base(handle):
    ptr, base = ipc_import(handle, 0)
    return base


class _DistComm:
    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def _gather_objects(self, obj):
        out = [None] * self.world
        self.dist.all_gather_object(out, obj, group=self.group)
        return out

    def pointer_tables(self, local: dict):
        return exchange_pointers(local, self.rank, self.world, self._gather_objects, ipc_export,
                                 _import_base)


class NcclComm(_DistComm):
    """All-gather and barriers on the current stream over an NCCL process group (one
    process per GPU): the ranks never synchronise the host within a step."""

    def __init__(self, group=None):
        super().__init__(group)
        self._word = torch.zeros(1, dtype=torch.int32, device="cuda")

    def all_gather(self, send, out):
        self.dist.all_gather_into_tensor(out.view(-1), send, group=self.group)

    def barrier(self):
        # an all-reduce of one word: no rank's later kernels start before every rank has
        # finished everything it enqueued before it
        self.dist.all_reduce(self._word, group=self.group)


class GlooComm(_DistComm):
    """All-gather and barriers through host memory over any process group: each
    exchange synchronises this process's device first."""

    @staticmethod
    def _sync():
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            torch.cuda.synchronize()

    def all_gather(self, send, out):
        self._sync()
        parts = [torch.zeros_like(send, device="cpu") for _ in range(self.world)]
        self.dist.all_gather(parts, send.cpu(), group=self.group)
        out.copy_(torch.stack(parts))

    def barrier(self):
        self._sync()
        self.dist.barrier(group=self.group)


class EPLayer:
    """One rank of the expert-parallel layer (one process per GPU).

    ``forward(logits, x)`` runs one step on this rank's T tokens and returns its [T,d]
    output; with ``backward=True`` the backward buffers are shared too and
    ``backward(dout)`` returns this rank's dx, dlogits and its home experts' weight
    gradients (replica gradients reduced back home).  Construction, ``forward`` and
    ``backward`` are collective: every rank calls them in the same order.  Weights are
    shared with the peers through the pointer tables: a caller that updates them in place
    must make every rank finish its step first."""

    def __init__(self, comm, T: int, E: int, k: int, S: int, W1, W3, W2, backward=False):
        self.comm = comm
        self.rank = EPRank(comm.rank, comm.world, T, E, k, S, W1, W3, W2)
        local = dict(self.rank.shared())
        if backward:
            local.update(self.rank.shared_backward())
        self.rank.tables, self._bases = comm.pointer_tables(local)

    def forward(self, logits, x):
        r = self.rank
        r.route(logits)
        self.comm.all_gather(r.send, r.gathered)
        r.plan_step()
        r.prefetch()
        r.dispatch(x)
        self.comm.barrier()
        r.ffn()
        self.comm.barrier()
        r.combine()
        return r.out

    def backward(self, dout):
        r = self.rank
        if "dy" not in r.tables:
            raise RuntimeError("EPLayer(..., backward=True) shares the backward buffers")
        r.bwd_combine(dout)
        self.comm.barrier()  # every rank's dy rows written
        r.bwd_ffn()
        self.comm.barrier()  # every rank's dx rows and partial gradients written
        r.bwd_reduce()
        r.bwd_dispatch()
        r.bwd_gates()
        return r.grads()

    def close(self):
        """Unmaps the peers' buffers (after every rank has finished its last step)."""
        for b in self._bases:
            ipc_close(b)
        self._bases = []


class LocalRanks:
    """W ranks of the expert-parallel layer inside one process on one GPU.

    Each rank's buffers are separate allocations; the pointer tables hold them directly;
    the all-gather is a copy of the stacked send vectors; the stages run rank by rank, so
    every rank's dispatch ends before any rank's FFN and every FFN before any combine,
    as the barriers order them across processes."""

    def __init__(self, ranks):
        self.ranks = list(ranks)
        tables = {name: [int(r.shared()[name].data_ptr()) for r in self.ranks] for name in SHARED}
        for r in self.ranks:
            r.tables = tables

    def stages(self, logits_shards, x_shards):
        """The step as (name, callable) pairs, each running one stage on every rank."""
        ranks = self.ranks

        def route():
            for r, lg in zip(ranks, logits_shards):
                r.route(lg)

        def plan():
            gathered = torch.stack([r.send for r in ranks])  # the all-gather
            for r in ranks:
                r.gathered.copy_(gathered)
                r.plan_step()

        def prefetch():
            for r in ranks:
                r.prefetch()

        def dispatch():
            for r, x in zip(ranks, x_shards):
                r.dispatch(x)

        def ffn():
            for r in ranks:
                r.ffn()

        def combine():
            for r in ranks:
                r.combine()

        return [("route", route), ("plan", plan), ("prefetch", prefetch), ("dispatch", dispatch),
                ("ffn", ffn), ("combine", combine)]

    def forward(self, logits_shards, x_shards):
        for _, f in self.stages(logits_shards, x_shards):
            f()
        return [r.out for r in self.ranks]

    def backward_stages(self, dout_shards):
        """The backward as (name, callable) pairs over every rank (buffers and tables set up
        here, before any stage runs)."""
        ranks = self.ranks
        if "dy" not in ranks[0].tables:
            tables = {name: [int(r.shared_backward()[name].data_ptr()) for r in ranks]
                      for name in SHARED_BWD}
            for r in ranks:
                r.tables = dict(r.tables, **tables)

        def combine():
            for r, g in zip(ranks, dout_shards):
                r.bwd_combine(g)

        def ffn():
            for r in ranks:
                r.bwd_ffn()

        def reduce_home():
            for r in ranks:
                r.bwd_reduce()

        def dispatch_and_gates():
            for r in ranks:
                r.bwd_dispatch()
                r.bwd_gates()

        return [("bwd_combine", combine), ("bwd_ffn", ffn), ("bwd_reduce_home", reduce_home),
                ("bwd_dispatch_gates", dispatch_and_gates)]

    def backward(self, dout_shards):
        """The backward of the last forward, stage by stage over the ranks; returns each
        rank's gradients (EPRank.grads)."""
        for _, f in self.backward_stages(dout_shards):
            f()
        return [r.grads() for r in self.ranks]
