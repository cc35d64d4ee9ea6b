"""Python binding of ``libmoe.so``: the MoE-layer hot path on one B200.

Argument marshalling only: each function below checks the tensors' dtype, device and
contiguity, passes raw device pointers and sizes to the C entry point of the same name
(declared in ``include/moe.h``) on the current CUDA stream, and raises on a non-zero host
status.  Every step of the path runs in the library's CUDA kernels; there is no CPU
fallback, and importing a function raises if the library has not been built.

``MoELayer`` owns the per-layer device buffers (PyTorch allocations) and runs the seven
calls in order: route, measure, plan, prefetch, dispatch, expert FFN, combine.  With
``fused=True`` the dispatch computes the row placement only and the expert FFN gathers its
rows from ``x`` (``moe_dispatch_index`` + ``moe_grouped_ffn_gather``).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK, MOE_ERR_ARG, MOE_ERR_SHAPE, MOE_ERR_LAUNCH, MOE_ERR_DEVICE = range(5)
DERR_NONFINITE, DERR_ID_RANGE, DERR_DUPLICATE, DERR_SLOTS, DERR_TIMEOUT = 1, 2, 4, 8, 16

ENTRY_POINTS = ("moe_topk", "moe_histogram_maxvio", "moe_plan_balanced", "moe_prefetch_replicas",
                "moe_dispatch", "moe_grouped_ffn", "moe_combine")
VARIANTS = ("moe_topk_biased", "moe_capacity_ledger", "moe_dispatch_capacity",
            "moe_grouped_ffn_capacity", "moe_combine_capacity")
FUSED = ("moe_dispatch_index", "moe_grouped_ffn_gather", "moe_route_plan",
         "moe_grouped_ffn_combine")
EXPERT_PARALLEL = ("moe_ep_counts", "moe_ep_plan", "moe_ep_prefetch", "moe_ep_dispatch",
                   "moe_ep_grouped_ffn", "moe_ep_combine", "moe_ipc_export", "moe_ipc_import",
                   "moe_ipc_close", "moe_ep_combine_backward", "moe_ep_grouped_ffn_backward",
                   "moe_ep_ffn_backward_workspace_bytes", "moe_ep_reduce_home",
                   "moe_ep_dispatch_backward")
BACKWARD = ("moe_combine_backward", "moe_grouped_ffn_backward", "moe_dispatch_backward",
            "moe_topk_backward")
HELPERS = ("moe_plan_get_layout", "moe_dispatch_workspace_words", "moe_status_string",
           "moe_set_ffn_tile_mode", "moe_ffn_tile_mode", "moe_ffn_pair_clusters",
           "moe_w2_to_f16")


class MoEError(RuntimeError):
    pass


class PlanLayout(ctypes.Structure):
    _fields_ = [("kept_rows", ctypes.c_int64), ("room_prefix", ctypes.c_int64),
                ("expert_home_off", ctypes.c_int64), ("stream_off", ctypes.c_int64),
                ("replica_expert", ctypes.c_int64), ("replica_list", ctypes.c_int64),
                ("n_groups", ctypes.c_int64), ("groups", ctypes.c_int64),
                ("words", ctypes.c_int64), ("max_groups_per_rank", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m load_balanced_dispatch_warp_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        sig = {
            "moe_topk": [P, I, I, I, P, P, P, P],
            "moe_histogram_maxvio": [P, I, I, I, I, P, P, P, P, P, P, P],
            "moe_plan_balanced": [P, I, I, I, I, I, P, P, P],
            "moe_prefetch_replicas": [P, P, P, P, I, I, I, I, I, P, P, P, P, P],
            "moe_dispatch": [P, P, P, I, I, I, I, I, I, P, P, P, P, P, P],
            "moe_grouped_ffn": [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P],
            "moe_combine": [P, P, P, I, I, I, P, P, P],
            "moe_topk_biased": [P, P, I, I, I, P, P, P, P],
            "moe_capacity_ledger": [P, I, I, I, I, I, P, P, P, P, P, P],
            "moe_selftest_bounded_wait": [P, I, P],
            "moe_dispatch_index": [P, P, I, I, I, I, I, P, P, P, P, P],
            "moe_grouped_ffn_gather": [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P],
            "moe_combine_backward": [P, P, P, P, I, I, I, P, P, P, P],
            "moe_grouped_ffn_backward": [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P,
                                         I64, P, P],
            "moe_dispatch_backward": [P, P, I, I, I, P, P, P],
            "moe_topk_backward": [P, P, P, I, I, I, P, P, P],
            "moe_route_plan": [P, P, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P],
            "moe_dispatch_capacity": [P, P, P, I, I, I, I, I, P, P, P, P, P, P],
            "moe_grouped_ffn_combine": [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P,
                                        P, P, P, P],
            "moe_grouped_ffn_capacity": [P, P, P, P, I, I, I, I, P, P, P, P],
            "moe_combine_capacity": [P, P, P, I, I, I, P, P, P],
            "moe_ep_counts": [P, I, I, I, P, P, P],
            "moe_ep_plan": [P, I, I, I, I, I, I, P, P, P, P, P, P, P, P],
            "moe_ep_prefetch": [P, P, P, P, I, I, I, I, I, I, P, P, P, P, P],
            "moe_ep_dispatch": [P, P, P, P, I, I, I, I, I, I, P, P, P, P, P],
            "moe_ep_grouped_ffn": [P, P, I, I, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, P],
            "moe_ep_combine": [P, P, P, I, I, I, I, P, P, P],
            "moe_ipc_export": [P, P, ctypes.POINTER(I64)],
            "moe_ipc_import": [P, I64, ctypes.POINTER(P), ctypes.POINTER(P)],
            "moe_ipc_close": [P],
            "moe_ep_combine_backward": [P, P, P, P, I, I, I, I, P, P, P, P],
            "moe_ep_grouped_ffn_backward": [P, P, P, I, I, P, P, P, P, P, P, I, I, I, I, I, I, P,
                                            P, P, P, P, P, I64, P, P],
            "moe_ep_reduce_home": [P, P, P, P, I, I, I, I, I, I, P, P],
            "moe_ep_dispatch_backward": [P, P, I, I, I, I, P, P, P],
            "moe_w2_to_f16": [P, I64, P, P],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.moe_plan_get_layout.argtypes = [I, I, I, ctypes.POINTER(PlanLayout)]
        L.moe_plan_get_layout.restype = ctypes.c_int
        L.moe_dispatch_workspace_words.argtypes = [I, I]
        L.moe_dispatch_workspace_words.restype = I64
        L.moe_capacity_rows.argtypes = [I, I, I, I, I]
        L.moe_capacity_rows.restype = I64
        L.moe_route_plan_workspace_words.argtypes = [I]
        L.moe_route_plan_workspace_words.restype = I64
        L.moe_ffn_backward_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
        L.moe_ffn_backward_workspace_bytes.restype = I64
        L.moe_ep_ffn_backward_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
        L.moe_ep_ffn_backward_workspace_bytes.restype = I64
        L.moe_set_ffn_tile_mode.argtypes = [I]
        L.moe_set_ffn_tile_mode.restype = I
        L.moe_ffn_tile_mode.argtypes = []
        L.moe_ffn_tile_mode.restype = I
        L.moe_ffn_pair_clusters.argtypes = []
        L.moe_ffn_pair_clusters.restype = I
        L.moe_status_string.argtypes = [I]
        L.moe_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoEError(f"{what}: {lib().moe_status_string(status).decode()} (status {status})")


def _ptr(t, dtype, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr() if t.numel() else None


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def plan_layout(E: int, R: int, S: int) -> PlanLayout:
    L = PlanLayout()
    _check(lib().moe_plan_get_layout(E, R, S, ctypes.byref(L)), "moe_plan_get_layout")
    return L


def dispatch_workspace_words(T: int, E: int) -> int:
    return int(lib().moe_dispatch_workspace_words(T, E))


# ----------------------------------------------------------------- the seven entry points
def moe_topk(logits, k, idx, gate, err, stream=None):
    T, E = logits.shape
    _check(lib().moe_topk(_ptr(logits, torch.float32, "logits"), T, E, k,
                          _ptr(idx, torch.int32, "idx"), _ptr(gate, torch.float32, "gate"),
                          _ptr(err, torch.int32, "err"), _stream(stream)), "moe_topk")


def moe_topk_biased(logits, bias, k, idx, gate, err, stream=None):
    T, E = logits.shape
    _check(lib().moe_topk_biased(_ptr(logits, torch.float32, "logits"), _ptr(bias, torch.float32, "bias"),
                                 T, E, k, _ptr(idx, torch.int32, "idx"), _ptr(gate, torch.float32, "gate"),
                                 _ptr(err, torch.int32, "err"), _stream(stream)), "moe_topk_biased")


def moe_capacity_ledger(counts, T, k, cf_num, cf_den, processed, overflow, padding, totals, err,
                        stream=None):
    E = counts.shape[0]
    i32 = torch.int32
    _check(lib().moe_capacity_ledger(
        _ptr(counts, i32, "counts"), T, k, E, cf_num, cf_den, _ptr(processed, i32, "processed"),
        _ptr(overflow, i32, "overflow"), _ptr(padding, i32, "padding"), _ptr(totals, i32, "totals"),
        _ptr(err, i32, "err"), _stream(stream)), "moe_capacity_ledger")


def set_ffn_tile_mode(mode: int) -> int:
    """Grouped-FFN tiling: 0 = one CTA per 128-row tile, 1 = 2-CTA clusters on 256-row tiles
    (tcgen05 cta_group::2).  Process-wide; returns the previous mode."""
    prev = int(lib().moe_ffn_tile_mode())
    _check(lib().moe_set_ffn_tile_mode(int(mode)), "moe_set_ffn_tile_mode")
    return prev


def ffn_pair_clusters() -> int:
    """2-CTA clusters the pair mode launches per GEMM on the current device (0 before use)."""
    return int(lib().moe_ffn_pair_clusters())


def moe_selftest_bounded_wait(err, limit_us=50000, stream=None):
    """Run the FFN's bounded wait on a barrier nothing arrives at (sets DERR_TIMEOUT)."""
    _check(lib().moe_selftest_bounded_wait(_ptr(err, torch.int32, "err"), int(limit_us), _stream(stream)),
           "moe_selftest_bounded_wait")


def route_plan_workspace_words(E: int) -> int:
    n = int(lib().moe_route_plan_workspace_words(E))
    if n < 0:
        raise MoEError(f"moe_route_plan_workspace_words: bad E={E}")
    return n


def moe_route_plan(logits, k, R, S, idx, gate, counts, loads, maxvio, balancedness, plan,
                   workspace, err, bias=None, stream=None):
    """moe_topk[_biased] + moe_histogram_maxvio (home map) + moe_plan_balanced in one launch."""
    T, E = logits.shape
    i32 = torch.int32
    if workspace.numel() < route_plan_workspace_words(E):
        raise ValueError("workspace smaller than moe_route_plan_workspace_words(E)")
    _check(lib().moe_route_plan(
        _ptr(logits, torch.float32, "logits"), _ptr(bias, torch.float32, "bias"), T, E, k, R, S,
        _ptr(idx, i32, "idx"), _ptr(gate, torch.float32, "gate"), _ptr(counts, i32, "counts"),
        _ptr(loads, i32, "loads"), _ptr(maxvio, torch.float64, "maxvio"),
        _ptr(balancedness, torch.float64, "balancedness"), _ptr(plan, i32, "plan"),
        _ptr(workspace, i32, "workspace"), _ptr(err, i32, "err"), _stream(stream)),
        "moe_route_plan")


def moe_histogram_maxvio(idx, E, R, counts, loads, maxvio, balancedness, err,
                         expert_to_rank=None, stream=None):
    T, k = idx.shape
    _check(lib().moe_histogram_maxvio(
        _ptr(idx, torch.int32, "idx"), T, k, E, R, _ptr(expert_to_rank, torch.int32, "expert_to_rank"),
        _ptr(counts, torch.int32, "counts"), _ptr(loads, torch.int32, "loads"),
        _ptr(maxvio, torch.float64, "maxvio"), _ptr(balancedness, torch.float64, "balancedness"),
        _ptr(err, torch.int32, "err"), _stream(stream)), "moe_histogram_maxvio")


def moe_plan_balanced(counts, T, k, R, S, plan, err, stream=None):
    E = counts.shape[0]
    _check(lib().moe_plan_balanced(_ptr(counts, torch.int32, "counts"), T, k, E, R, S,
                                   _ptr(plan, torch.int32, "plan"), _ptr(err, torch.int32, "err"),
                                   _stream(stream)), "moe_plan_balanced")


def moe_prefetch_replicas(plan, W1, W3, W2, R, S, P1, P3, P2, err, stream=None):
    E, F, d = W1.shape
    bf, hf = torch.bfloat16, torch.float16
    _check(lib().moe_prefetch_replicas(
        _ptr(plan, torch.int32, "plan"), _ptr(W1, bf, "W1"), _ptr(W3, bf, "W3"), _ptr(W2, hf, "W2"),
        E, R, S, d, F, _ptr(P1, bf, "P1"), _ptr(P3, bf, "P3"), _ptr(P2, hf, "P2"),
        _ptr(err, torch.int32, "err"), _stream(stream)), "moe_prefetch_replicas")


def moe_dispatch(x, idx, plan, E, R, S, workspace, recv, perm, src, err, stream=None):
    T, d = x.shape
    k = idx.shape[1]
    _check(lib().moe_dispatch(
        _ptr(x, torch.bfloat16, "x"), _ptr(idx, torch.int32, "idx"), _ptr(plan, torch.int32, "plan"),
        T, k, E, R, S, d, _ptr(workspace, torch.int32, "workspace"), _ptr(recv, torch.bfloat16, "recv"),
        _ptr(perm, torch.int32, "perm"), _ptr(src, torch.int32, "src"), _ptr(err, torch.int32, "err"),
        _stream(stream)), "moe_dispatch")


NOALLOC_SCRATCH_WORDS = 524288  # MOE_NOALLOC_SCRATCH_WORDS


def moe_dispatch_noalloc(x, idx, plan, E, R, S, recv, perm, src, err, stream=None):
    """moe_dispatch without a workspace: for callers that cannot allocate device memory
    when they dispatch; the library uses its own static 2 MiB scratch (see moe.h)."""
    f = lib().moe_dispatch_noalloc
    if f.restype is not ctypes.c_int or f.argtypes is None:
        P, I = ctypes.c_void_p, ctypes.c_int
        f.argtypes = [P, P, P, I, I, I, I, I, I, P, P, P, P, P]
        f.restype = ctypes.c_int
    T, d = x.shape
    k = idx.shape[1]
    _check(f(_ptr(x, torch.bfloat16, "x"), _ptr(idx, torch.int32, "idx"), _ptr(plan, torch.int32, "plan"),
             T, k, E, R, S, d, _ptr(recv, torch.bfloat16, "recv"), _ptr(perm, torch.int32, "perm"),
             _ptr(src, torch.int32, "src"), _ptr(err, torch.int32, "err"), _stream(stream)),
           "moe_dispatch_noalloc")


def moe_grouped_ffn(recv, plan, W1, W3, W2, P1, P3, P2, T, k, R, S, h, y, err, stream=None):
    E, F, d = W1.shape
    bf, hf = torch.bfloat16, torch.float16
    _check(lib().moe_grouped_ffn(
        _ptr(recv, bf, "recv"), _ptr(plan, torch.int32, "plan"), _ptr(W1, bf, "W1"),
        _ptr(W3, bf, "W3"), _ptr(W2, hf, "W2"), _ptr(P1, bf, "P1"), _ptr(P3, bf, "P3"),
        _ptr(P2, hf, "P2"), T, k, E, R, S, d, F, _ptr(h, hf, "h"), _ptr(y, bf, "y"),
        _ptr(err, torch.int32, "err"), _stream(stream)), "moe_grouped_ffn")


def moe_dispatch_index(idx, plan, E, R, S, workspace, perm, src, err, stream=None):
    """moe_dispatch without the row copy: perm and src only (for moe_grouped_ffn_gather)."""
    T, k = idx.shape
    _check(lib().moe_dispatch_index(
        _ptr(idx, torch.int32, "idx"), _ptr(plan, torch.int32, "plan"), T, k, E, R, S,
        _ptr(workspace, torch.int32, "workspace"), _ptr(perm, torch.int32, "perm"),
        _ptr(src, torch.int32, "src"), _ptr(err, torch.int32, "err"), _stream(stream)),
        "moe_dispatch_index")


def moe_grouped_ffn_gather(x, src, plan, W1, W3, W2, P1, P3, P2, T, k, R, S, h, y, err,
                           stream=None):
    """moe_grouped_ffn with GEMM 1's rows gathered as x[src[row]] (no recv buffer)."""
    E, F, d = W1.shape
    bf, hf = torch.bfloat16, torch.float16
    _check(lib().moe_grouped_ffn_gather(
        _ptr(x, bf, "x"), _ptr(src, torch.int32, "src"), _ptr(plan, torch.int32, "plan"),
        _ptr(W1, bf, "W1"), _ptr(W3, bf, "W3"), _ptr(W2, hf, "W2"), _ptr(P1, bf, "P1"),
        _ptr(P3, bf, "P3"), _ptr(P2, hf, "P2"), T, k, E, R, S, d, F, _ptr(h, hf, "h"),
        _ptr(y, bf, "y"), _ptr(err, torch.int32, "err"), _stream(stream)),
        "moe_grouped_ffn_gather")


# ----------------------------------------------------------------- fixed-capacity mode
def capacity_rows(T: int, k: int, E: int, cf_num: int = 5, cf_den: int = 4) -> int:
    """cap = ceil(T*k / E * cf_num / cf_den) rows per expert (moe_capacity_rows)."""
    cap = int(lib().moe_capacity_rows(T, k, E, cf_num, cf_den))
    if cap < 0:
        raise MoEError("moe_capacity_rows: non-positive argument")
    return cap


def moe_dispatch_capacity(x, idx, counts, cap, workspace, recv, perm, src, err, stream=None):
    """Each expert keeps its first cap assignments (token order) in rows [e*cap, (e+1)*cap);
    the rest are dropped (perm -1); padding rows are zero with src -1."""
    T, d = x.shape
    k = idx.shape[1]
    E = counts.shape[0]
    _check(lib().moe_dispatch_capacity(
        _ptr(x, torch.bfloat16, "x"), _ptr(idx, torch.int32, "idx"),
        _ptr(counts, torch.int32, "counts"), T, k, E, cap, d,
        _ptr(workspace, torch.int32, "workspace"), _ptr(recv, torch.bfloat16, "recv"),
        _ptr(perm, torch.int32, "perm"), _ptr(src, torch.int32, "src"),
        _ptr(err, torch.int32, "err"), _stream(stream)), "moe_dispatch_capacity")


def moe_grouped_ffn_capacity(recv, W1, W3, W2, cap, h, y, err, stream=None):
    E, F, d = W1.shape
    bf, hf = torch.bfloat16, torch.float16
    _check(lib().moe_grouped_ffn_capacity(
        _ptr(recv, bf, "recv"), _ptr(W1, bf, "W1"), _ptr(W3, bf, "W3"), _ptr(W2, hf, "W2"), E, cap,
        d, F, _ptr(h, hf, "h"), _ptr(y, bf, "y"), _ptr(err, torch.int32, "err"), _stream(stream)),
        "moe_grouped_ffn_capacity")


def moe_combine_capacity(y, perm, gate, out, err, stream=None):
    T, k = perm.shape
    d = out.shape[1]
    _check(lib().moe_combine_capacity(
        _ptr(y, torch.bfloat16, "y"), _ptr(perm, torch.int32, "perm"),
        _ptr(gate, torch.float32, "gate"), T, k, d, _ptr(out, torch.bfloat16, "out"),
        _ptr(err, torch.int32, "err"), _stream(stream)), "moe_combine_capacity")


class CapacityLayer:
    """The fixed-capacity (dropping) mode of one MoE layer: per-layer device buffers and the
    calls in order -- moe_topk, moe_histogram_maxvio (raw demand, before any exclusion),
    moe_capacity_ledger, moe_dispatch_capacity, moe_grouped_ffn_capacity,
    moe_combine_capacity."""

    def __init__(self, T, E, k, d, F, cf_num=5, cf_den=4, device="cuda"):
        self.T, self.E, self.k, self.d, self.F = T, E, k, d, F
        self.cf = (cf_num, cf_den)
        self.cap = capacity_rows(T, k, E, cf_num, cf_den)
        i32, dev = torch.int32, device
        rows = E * self.cap
        self.idx = torch.empty(T, k, dtype=i32, device=dev)
        self.gate = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=i32, device=dev)
        self.loads = torch.empty(1, dtype=i32, device=dev)
        self.maxvio = torch.empty(1, dtype=torch.float64, device=dev)
        self.balancedness = torch.empty(1, dtype=torch.float64, device=dev)
        self.processed = torch.empty(E, dtype=i32, device=dev)
        self.overflow = torch.empty(E, dtype=i32, device=dev)
        self.padding = torch.empty(E, dtype=i32, device=dev)
        self.totals = torch.empty(4, dtype=i32, device=dev)
        self.workspace = torch.empty(max(1, dispatch_workspace_words(T, E)), dtype=i32, device=dev)
        self.recv = torch.empty(rows, d, dtype=torch.bfloat16, device=dev)
        self.perm = torch.empty(T, k, dtype=i32, device=dev)
        self.src = torch.empty(rows, dtype=i32, device=dev)
        self.h = torch.empty(rows, F, dtype=torch.float16, device=dev)
        self.y = torch.empty(rows, d, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
        self.err = torch.zeros(1, dtype=i32, device=dev)

    def forward(self, logits, x, W1, W3, W2, stream=None):
        moe_topk(logits, self.k, self.idx, self.gate, self.err, stream)
        moe_histogram_maxvio(self.idx, self.E, 1, self.counts, self.loads, self.maxvio,
                             self.balancedness, self.err, stream=stream)
        moe_capacity_ledger(self.counts, self.T, self.k, self.cf[0], self.cf[1], self.processed,
                            self.overflow, self.padding, self.totals, self.err, stream)
        moe_dispatch_capacity(x, self.idx, self.counts, self.cap, self.workspace, self.recv,
                              self.perm, self.src, self.err, stream)
        moe_grouped_ffn_capacity(self.recv, W1, W3, W2, self.cap, self.h, self.y, self.err, stream)
        moe_combine_capacity(self.y, self.perm, self.gate, self.out, self.err, stream)
        return self.out


def moe_grouped_ffn_combine(recv, plan, W1, W3, W2, P1, P3, P2, src, perm, gate, R, S, h, out32,
                            out, err, stream=None):
    """moe_grouped_ffn + moe_combine with the gate-weighted sum in GEMM 2's epilogue (fp32
    atomics into the scratch out32 [T,d], then bf16 into out): no y buffer, no combine
    kernel."""
    E, F, d = W1.shape
    T, k = perm.shape
    bf, hf, i32 = torch.bfloat16, torch.float16, torch.int32
    _check(lib().moe_grouped_ffn_combine(
        _ptr(recv, bf, "recv"), _ptr(plan, i32, "plan"), _ptr(W1, bf, "W1"), _ptr(W3, bf, "W3"),
        _ptr(W2, hf, "W2"), _ptr(P1, bf, "P1"), _ptr(P3, bf, "P3"), _ptr(P2, hf, "P2"),
        _ptr(src, i32, "src"), _ptr(perm, i32, "perm"), _ptr(gate, torch.float32, "gate"), T, k,
        E, R, S, d, F, _ptr(h, hf, "h"), _ptr(out32, torch.float32, "out32"), _ptr(out, bf, "out"),
        _ptr(err, i32, "err"), _stream(stream)), "moe_grouped_ffn_combine")


# ------------------------------------------------------- expert parallelism across GPUs
EP_MAX_RANKS = 64           # MOE_EP_MAX_RANKS
IPC_HANDLE_BYTES = 64       # MOE_IPC_HANDLE_BYTES


def _table(ptrs, name, rows=1):
    """A host array of device pointers (one per rank) for the *_ranks arguments.  With no
    rows to move (rows == 0: empty buffers, null pointers) the calls do not read it."""
    ptrs = [int(p) for p in ptrs]
    if not ptrs or (rows and any(p == 0 for p in ptrs)):
        raise ValueError(f"{name}: one non-null device pointer per rank")
    return (ctypes.c_void_p * len(ptrs))(*ptrs)


def moe_ep_counts(idx, E, err, send, stream=None):
    T, k = idx.shape
    _check(lib().moe_ep_counts(_ptr(idx, torch.int32, "idx"), T, k, E, _ptr(err, torch.int32, "err"),
                               _ptr(send, torch.int32, "send"), _stream(stream)), "moe_ep_counts")


def moe_ep_plan(gathered, me, T, k, S, counts, q_base, loads, maxvio, balancedness, plan, err,
                stream=None):
    W, E1 = gathered.shape
    i32 = torch.int32
    _check(lib().moe_ep_plan(
        _ptr(gathered, i32, "gathered"), W, me, T, k, E1 - 1, S, _ptr(counts, i32, "counts"),
        _ptr(q_base, i32, "q_base"), _ptr(loads, i32, "loads"), _ptr(maxvio, torch.float64, "maxvio"),
        _ptr(balancedness, torch.float64, "balancedness"), _ptr(plan, i32, "plan"),
        _ptr(err, i32, "err"), _stream(stream)), "moe_ep_plan")


def moe_ep_prefetch(plan, W1_ranks, W3_ranks, W2_ranks, me, E, S, d, F, P1, P3, P2, err,
                    stream=None):
    W = len(W1_ranks)
    bf, hf = torch.bfloat16, torch.float16
    _check(lib().moe_ep_prefetch(
        _ptr(plan, torch.int32, "plan"), _table(W1_ranks, "W1_ranks"), _table(W3_ranks, "W3_ranks"),
        _table(W2_ranks, "W2_ranks"), W, me, E, S, d, F, _ptr(P1, bf, "P1"), _ptr(P3, bf, "P3"),
        _ptr(P2, hf, "P2"), _ptr(err, torch.int32, "err"), _stream(stream)), "moe_ep_prefetch")


def moe_ep_dispatch(x, idx, q_base, plan, E, S, workspace, recv_ranks, perm, err, stream=None):
    T, d = x.shape
    k = idx.shape[1]
    i32 = torch.int32
    _check(lib().moe_ep_dispatch(
        _ptr(x, torch.bfloat16, "x"), _ptr(idx, i32, "idx"), _ptr(q_base, i32, "q_base"),
        _ptr(plan, i32, "plan"), len(recv_ranks), T, k, E, S, d,
        _ptr(workspace, i32, "workspace"), _table(recv_ranks, "recv_ranks", T),
        _ptr(perm, i32, "perm"), _ptr(err, i32, "err"), _stream(stream)), "moe_ep_dispatch")


def moe_ep_grouped_ffn(recv, plan, W, me, W1, W3, W2, P1, P3, P2, T, k, E, S, groups_ws, h, y,
                       err, stream=None):
    _, F, d = W1.shape
    bf, hf = torch.bfloat16, torch.float16
    _check(lib().moe_ep_grouped_ffn(
        _ptr(recv, bf, "recv"), _ptr(plan, torch.int32, "plan"), W, me, _ptr(W1, bf, "W1"),
        _ptr(W3, bf, "W3"), _ptr(W2, hf, "W2"), _ptr(P1, bf, "P1"), _ptr(P3, bf, "P3"),
        _ptr(P2, hf, "P2"), T, k, E, S, d, F, _ptr(groups_ws, torch.int32, "groups_ws"),
        _ptr(h, hf, "h"), _ptr(y, bf, "y"), _ptr(err, torch.int32, "err"), _stream(stream)),
        "moe_ep_grouped_ffn")


def moe_ep_combine(y_ranks, perm, gate, d, out, err, stream=None):
    T, k = perm.shape
    _check(lib().moe_ep_combine(
        _table(y_ranks, "y_ranks", T), _ptr(perm, torch.int32, "perm"), _ptr(gate, torch.float32, "gate"),
        len(y_ranks), T, k, d, _ptr(out, torch.bfloat16, "out"), _ptr(err, torch.int32, "err"),
        _stream(stream)), "moe_ep_combine")


def moe_ep_combine_backward(dout, y_ranks, perm, gate, dy_ranks, dgate, err, stream=None):
    T, k = perm.shape
    _check(lib().moe_ep_combine_backward(
        _ptr(dout, torch.bfloat16, "dout"), _table(y_ranks, "y_ranks", T), _ptr(perm, torch.int32, "perm"),
        _ptr(gate, torch.float32, "gate"), len(y_ranks), T, k, dout.shape[1],
        _table(dy_ranks, "dy_ranks", T), _ptr(dgate, torch.float32, "dgate"),
        _ptr(err, torch.int32, "err"), _stream(stream)), "moe_ep_combine_backward")


def ep_ffn_backward_workspace_bytes(T, k, E, W, S, d, F) -> int:
    n = int(lib().moe_ep_ffn_backward_workspace_bytes(T, k, E, W, S, d, F))
    if n < 0:
        raise MoEError("moe_ep_ffn_backward_workspace_bytes: invalid shape")
    return n


def moe_ep_grouped_ffn_backward(recv, dy, plan, W, me, W1, W3, W2, P1, P3, P2, T, k, E, S,
                                groups_ws, dx_rows, dP1, dP3, dP2, workspace, err, stream=None):
    _, F, d = W1.shape
    bf, hf, f32 = torch.bfloat16, torch.float16, torch.float32
    if workspace.dtype != torch.uint8 or not workspace.is_cuda:
        raise TypeError("workspace must be a CUDA uint8 tensor")
    _check(lib().moe_ep_grouped_ffn_backward(
        _ptr(recv, bf, "recv"), _ptr(dy, bf, "dy"), _ptr(plan, torch.int32, "plan"), W, me,
        _ptr(W1, bf, "W1"), _ptr(W3, bf, "W3"), _ptr(W2, hf, "W2"), _ptr(P1, bf, "P1"),
        _ptr(P3, bf, "P3"), _ptr(P2, hf, "P2"), T, k, E, S, d, F,
        _ptr(groups_ws, torch.int32, "groups_ws"), _ptr(dx_rows, bf, "dx_rows"),
        _ptr(dP1, f32, "dP1"), _ptr(dP3, f32, "dP3"), _ptr(dP2, f32, "dP2"),
        workspace.data_ptr(), workspace.numel(), _ptr(err, torch.int32, "err"), _stream(stream)),
        "moe_ep_grouped_ffn_backward")


def moe_ep_reduce_home(plan, dP1_ranks, dP3_ranks, dP2_ranks, me, E, S, d, F, err,
                       stream=None):
    _check(lib().moe_ep_reduce_home(
        _ptr(plan, torch.int32, "plan"), _table(dP1_ranks, "dP1_ranks"),
        _table(dP3_ranks, "dP3_ranks"), _table(dP2_ranks, "dP2_ranks"), len(dP1_ranks), me, E,
        S, d, F, _ptr(err, torch.int32, "err"), _stream(stream)), "moe_ep_reduce_home")


def moe_ep_dispatch_backward(dx_rows_ranks, perm, d, dx, err, stream=None):
    T, k = perm.shape
    _check(lib().moe_ep_dispatch_backward(
        _table(dx_rows_ranks, "dx_rows_ranks", T), _ptr(perm, torch.int32, "perm"),
        len(dx_rows_ranks), T, k, d, _ptr(dx, torch.bfloat16, "dx"), _ptr(err, torch.int32, "err"),
        _stream(stream)), "moe_ep_dispatch_backward")


def ipc_export(t: torch.Tensor):
    """(handle bytes, offset) naming the allocation that holds tensor t's storage."""
    if not t.is_cuda:
        raise TypeError("ipc_export needs a CUDA tensor")
    h = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_int64(0)
    _check(lib().moe_ipc_export(t.data_ptr(), h, ctypes.byref(off)), "moe_ipc_export")
    return h.raw, off.value


def ipc_import(handle: bytes, offset: int):
    """(device pointer, mapping base) of another process's exported buffer."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("IPC handle of the wrong size")
    ptr, base = ctypes.c_void_p(), ctypes.c_void_p()
    buf = ctypes.create_string_buffer(handle, IPC_HANDLE_BYTES)
    _check(lib().moe_ipc_import(buf, offset, ctypes.byref(ptr), ctypes.byref(base)),
           "moe_ipc_import")
    return ptr.value, base.value


def ipc_close(base: int):
    _check(lib().moe_ipc_close(base), "moe_ipc_close")


def w2_to_f16(W2_bf16, out=None, stream=None):
    """The fp16 copy of a bf16 down projection (once per weight version): moe_w2_to_f16."""
    if out is None:
        out = torch.empty(W2_bf16.shape, dtype=torch.float16, device=W2_bf16.device)
    if out.shape != W2_bf16.shape:
        raise ValueError("out must have W2's shape")
    _check(lib().moe_w2_to_f16(_ptr(W2_bf16, torch.bfloat16, "W2_bf16"), W2_bf16.numel(),
                               _ptr(out, torch.float16, "out"), _stream(stream)), "moe_w2_to_f16")
    return out


def moe_combine(y, perm, gate, out, err, stream=None):
    T, k = perm.shape
    d = out.shape[1]
    _check(lib().moe_combine(_ptr(y, torch.bfloat16, "y"), _ptr(perm, torch.int32, "perm"),
                             _ptr(gate, torch.float32, "gate"), T, k, d,
                             _ptr(out, torch.bfloat16, "out"), _ptr(err, torch.int32, "err"),
                             _stream(stream)), "moe_combine")


# ----------------------------------------------------------------- backward pass
def ffn_backward_workspace_bytes(T, k, E, R, S, d, F) -> int:
    n = int(lib().moe_ffn_backward_workspace_bytes(T, k, E, R, S, d, F))
    if n < 0:
        raise MoEError("moe_ffn_backward_workspace_bytes: invalid shape")
    return n


def moe_combine_backward(dout, y, perm, gate, dy, dgate, err, stream=None):
    T, k = perm.shape
    d = dout.shape[1]
    _check(lib().moe_combine_backward(
        _ptr(dout, torch.bfloat16, "dout"), _ptr(y, torch.bfloat16, "y"), _ptr(perm, torch.int32, "perm"),
        _ptr(gate, torch.float32, "gate"), T, k, d, _ptr(dy, torch.bfloat16, "dy"),
        _ptr(dgate, torch.float32, "dgate"), _ptr(err, torch.int32, "err"), _stream(stream)),
        "moe_combine_backward")


def moe_grouped_ffn_backward(recv, dy, h, plan, W1, W3, W2, T, k, R, S, dx_rows, dW1, dW3, dW2,
                             workspace, err, stream=None):
    E, F, d = W1.shape
    bf, hf, f32 = torch.bfloat16, torch.float16, torch.float32
    _check(lib().moe_grouped_ffn_backward(
        _ptr(recv, bf, "recv"), _ptr(dy, bf, "dy"), _ptr(h, hf, "h"), _ptr(plan, torch.int32, "plan"),
        _ptr(W1, bf, "W1"), _ptr(W3, bf, "W3"), _ptr(W2, hf, "W2"), T, k, E, R, S, d, F,
        _ptr(dx_rows, bf, "dx_rows"), _ptr(dW1, f32, "dW1"), _ptr(dW3, f32, "dW3"),
        _ptr(dW2, f32, "dW2"), _ptr(workspace, torch.uint8, "workspace"),
        workspace.numel() if workspace is not None else 0, _ptr(err, torch.int32, "err"),
        _stream(stream)), "moe_grouped_ffn_backward")


def moe_dispatch_backward(dx_rows, perm, dx, err, stream=None):
    T, k = perm.shape
    d = dx.shape[1]
    _check(lib().moe_dispatch_backward(
        _ptr(dx_rows, torch.bfloat16, "dx_rows"), _ptr(perm, torch.int32, "perm"), T, k, d,
        _ptr(dx, torch.bfloat16, "dx"), _ptr(err, torch.int32, "err"), _stream(stream)),
        "moe_dispatch_backward")


def moe_topk_backward(gate, dgate, idx, E, dlogits, err, stream=None):
    T, k = idx.shape
    _check(lib().moe_topk_backward(
        _ptr(gate, torch.float32, "gate"), _ptr(dgate, torch.float32, "dgate"),
        _ptr(idx, torch.int32, "idx"), T, E, k, _ptr(dlogits, torch.float32, "dlogits"),
        _ptr(err, torch.int32, "err"), _stream(stream)), "moe_topk_backward")


# ----------------------------------------------------------------- one layer
class MoELayer:
    """Device buffers of one MoE layer of shape (T, E, k, R, S, d, F) and the seven calls.

    The replica pool (P1, P3, P2: R*S slots) is allocated once here; several layers may
    share one pool by passing ``pool=`` (it is process-global in the MoonEP design).
    ``fused=True``: no recv buffer; the FFN gathers the rows of the ``x`` last dispatched.
    ``fused_combine=True``: no y buffer; GEMM 2's epilogue adds the gate-weighted rows into
    an fp32 [T,d] scratch (``out32``), converted to ``out`` in the same call
    (``moe_grouped_ffn_combine``); ``combine()`` then has nothing left to do.
    """

    def __init__(self, T, E, k, R, S, d, F, device="cuda", pool=None, fused=False,
                 fused_combine=False):
        self.T, self.E, self.k, self.R, self.S, self.d, self.F = T, E, k, R, S, d, F
        self.fused = bool(fused)
        self.fused_combine = bool(fused_combine)
        if self.fused and self.fused_combine:
            raise ValueError("fused (gathering GEMM 1) and fused_combine are separate options")
        self._x = None
        self.A = T * k
        self.C = self.A // R
        dev = torch.device(device)
        i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
        self.layout = plan_layout(E, R, S)
        self.idx = torch.empty(T, k, dtype=i32, device=dev)
        self.gate = torch.empty(T, k, dtype=f32, device=dev)
        self.err = torch.zeros(1, dtype=i32, device=dev)
        self.counts = torch.empty(E, dtype=i32, device=dev)
        self.loads = torch.empty(R, dtype=i32, device=dev)
        self.maxvio = torch.empty(1, dtype=torch.float64, device=dev)
        self.balancedness = torch.empty(1, dtype=torch.float64, device=dev)
        self.plan = torch.empty(self.layout.words, dtype=i32, device=dev)
        self.workspace = torch.empty(max(1, dispatch_workspace_words(T, E)), dtype=i32, device=dev)
        self.rp_workspace = torch.empty(route_plan_workspace_words(E), dtype=i32, device=dev)
        self.recv = None if self.fused else torch.empty(self.A, d, dtype=bf, device=dev)
        self.perm = torch.empty(T, k, dtype=i32, device=dev)
        self.src = torch.empty(self.A, dtype=i32, device=dev)
        self.h = torch.empty(self.A, F, dtype=torch.float16, device=dev)
        self.y = None if self.fused_combine else torch.empty(self.A, d, dtype=bf, device=dev)
        self.out32 = torch.empty(T, d, dtype=f32, device=dev) if self.fused_combine else None
        self.out = torch.empty(T, d, dtype=bf, device=dev)
        if pool is None and S > 0:
            pool = (torch.empty(R * S, F, d, dtype=bf, device=dev),
                    torch.empty(R * S, F, d, dtype=bf, device=dev),
                    torch.empty(R * S, d, F, dtype=torch.float16, device=dev))
        self.pool = pool if S > 0 else (None, None, None)

    def plan_field(self, name):
        L = self.layout
        sizes = dict(kept_rows=self.R, room_prefix=self.R + 1, expert_home_off=self.E,
                     stream_off=self.E + 1, replica_expert=self.R * self.S,
                     replica_list=1 + self.R * self.S, n_groups=self.R,
                     groups=self.R * L.max_groups_per_rank * 4)
        off = getattr(L, name)
        return self.plan[off:off + sizes[name]]

    # each step on its own (the caller orders them)
    def route(self, logits, stream=None):
        moe_topk(logits, self.k, self.idx, self.gate, self.err, stream)

    def measure(self, expert_to_rank=None, stream=None):
        moe_histogram_maxvio(self.idx, self.E, self.R, self.counts, self.loads, self.maxvio,
                             self.balancedness, self.err, expert_to_rank, stream)

    def balance(self, stream=None):
        moe_plan_balanced(self.counts, self.T, self.k, self.R, self.S, self.plan, self.err, stream)

    def prefetch(self, W1, W3, W2, stream=None):
        P1, P3, P2 = self.pool
        moe_prefetch_replicas(self.plan, W1, W3, W2, self.R, self.S, P1, P3, P2, self.err, stream)

    def dispatch(self, x, stream=None):
        if self.fused:
            if x.shape != (self.T, self.d) or x.dtype != torch.bfloat16:
                raise ValueError("x must be [T,d] bf16")
            self._x = x
            moe_dispatch_index(self.idx, self.plan, self.E, self.R, self.S, self.workspace,
                               self.perm, self.src, self.err, stream)
        else:
            moe_dispatch(x, self.idx, self.plan, self.E, self.R, self.S, self.workspace,
                         self.recv, self.perm, self.src, self.err, stream)

    def expert_ffn(self, W1, W3, W2, stream=None):
        P1, P3, P2 = self.pool
        if self.fused_combine:
            moe_grouped_ffn_combine(self.recv, self.plan, W1, W3, W2, P1, P3, P2, self.src,
                                    self.perm, self.gate, self.R, self.S, self.h, self.out32,
                                    self.out, self.err, stream)
        elif self.fused:
            if self._x is None:
                raise RuntimeError("fused expert_ffn needs a dispatch(x) first")
            moe_grouped_ffn_gather(self._x, self.src, self.plan, W1, W3, W2, P1, P3, P2, self.T,
                                   self.k, self.R, self.S, self.h, self.y, self.err, stream)
        else:
            moe_grouped_ffn(self.recv, self.plan, W1, W3, W2, P1, P3, P2, self.T, self.k,
                            self.R, self.S, self.h, self.y, self.err, stream)

    def combine(self, stream=None):
        if self.fused_combine:
            return  # done in the expert FFN's epilogue
        moe_combine(self.y, self.perm, self.gate, self.out, self.err, stream)

    def route_plan(self, logits, stream=None):
        """route + measure (home map) + balance as one fused launch (same outputs)."""
        moe_route_plan(logits, self.k, self.R, self.S, self.idx, self.gate, self.counts,
                       self.loads, self.maxvio, self.balancedness, self.plan, self.rp_workspace,
                       self.err, stream=stream)

    def forward(self, logits, x, W1, W3, W2, stream=None):
        """The whole path on the current stream: routing, histogram and plan fused
        (``route_plan``), prefetch, dispatch, the grouped FFN, the combine; returns ``out``
        [T,d] bf16 (device)."""
        self.route_plan(logits, stream)
        self.prefetch(W1, W3, W2, stream)
        self.dispatch(x, stream)
        self.expert_ffn(W1, W3, W2, stream)
        self.combine(stream)
        return self.out

    def backward(self, dout, W1, W3, W2, stream=None):
        """Backward of the last forward() (unfused layers: it reads recv, y and h):
        dout [T,d] bf16 -> dict(dx [T,d] bf16, dlogits [T,E] fp32, dW1, dW3 [E,F,d] fp32,
        dW2 [E,d,F] fp32).  Buffers are allocated on first use and reused."""
        if self.fused or self.fused_combine:
            raise RuntimeError("backward needs the dispatched rows and y: use an unfused layer")
        if not hasattr(self, "_bwd"):
            dev = self.idx.device
            T, E, k, d, F, A = self.T, self.E, self.k, self.d, self.F, self.A
            f32 = torch.float32
            ws = ffn_backward_workspace_bytes(T, k, E, self.R, self.S, d, F)
            self._bwd = dict(
                dy=torch.empty(A, d, dtype=torch.bfloat16, device=dev),
                dgate=torch.empty(T, k, dtype=f32, device=dev),
                dx_rows=torch.empty(A, d, dtype=torch.bfloat16, device=dev),
                dx=torch.empty(T, d, dtype=torch.bfloat16, device=dev),
                dlogits=torch.empty(T, E, dtype=f32, device=dev),
                dW1=torch.empty(E, F, d, dtype=f32, device=dev),
                dW3=torch.empty(E, F, d, dtype=f32, device=dev),
                dW2=torch.empty(E, d, F, dtype=f32, device=dev),
                workspace=torch.empty(max(ws, 256), dtype=torch.uint8, device=dev))
        b = self._bwd
        moe_combine_backward(dout, self.y, self.perm, self.gate, b["dy"], b["dgate"], self.err, stream)
        moe_grouped_ffn_backward(self.recv, b["dy"], self.h, self.plan, W1, W3, W2, self.T, self.k,
                                 self.R, self.S, b["dx_rows"], b["dW1"], b["dW3"], b["dW2"],
                                 b["workspace"], self.err, stream)
        moe_dispatch_backward(b["dx_rows"], self.perm, b["dx"], self.err, stream)
        moe_topk_backward(self.gate, b["dgate"], self.idx, self.E, b["dlogits"], self.err, stream)
        return b

    # kernels launched by forward() (for launch accounting)
    def kernels_per_forward(self) -> int:
        n = 2                                 # reset (err, workspace); routing + histogram + plan
        n += 1 if self.S > 0 else 0           # prefetch
        n += (2 if self.fused else 3) if self.T > 0 else 0  # workspace reset, ranks[, row scatter]
        n += 2 if self.T > 0 else 0           # two grouped GEMMs
        n += 1 if self.T > 0 else 0           # combine (fused: the fp32 -> bf16 pass)
        return n
