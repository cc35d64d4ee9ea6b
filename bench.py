"""Throughput of the MoE-layer hot path on B200: one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one pass of the whole path (top-k, histogram/maxvio, balanced plan, replica
prefetch, dispatch, grouped SwiGLU FFN, combine) over one batch of seeded synthetic
inputs already resident in HBM.  The default workload is the near-balanced fine-grained
layer (4096 tokens, 64 experts, top-6, 8 simulated ranks, 8 slots, d=2048, F=1408).
Under torchrun (N > 1) every rank runs an independent replica of the same layer on its
own GPU (no collective on the data path); timing is the max over ranks.

`--impl reference` times the CPU oracle instead (rank 0 only), on a bounded sample of the
same workload per step.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from load_balanced_dispatch_warp_b200 import inputs as I  # noqa: E402

METRIC = "MoE layer tokens/s"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) per call of the dominant call (both grouped-FFN kernels) from
# an ncu capture (profiles/ffn_kernel_near_balanced.md), keyed by workload, tile mode and
# kernel sources hash: it reads null as soon as the kernel sources change.
TRAFFIC = {"near_balanced:0:d4ffa6ea7d84948f": int((926.897408 + 63.862528 + 478.883328 + 81.526272) * 1e6)}


def sources_hash() -> str:
    """Hash of the grouped-FFN kernel's device code: grouped_ffn.cu and the device-side
    helpers of common.cuh (host declarations there do not change the kernel)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "load_balanced_dispatch_warp_b200", "csrc")
    with open(os.path.join(csrc, "grouped_ffn.cu"), "rb") as fh:
        h.update(fh.read())
    with open(os.path.join(csrc, "common.cuh"), "rb") as fh:
        text = fh.read()
    h.update(text[text.index(b"device side"):])
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        return self.summarize(out)

    @staticmethod
    def summarize(out: str) -> dict:
        """Clock record from `nvidia-smi --query-gpu=QUERY --format=csv,noheader,nounits`
        lines: the median SM clock over the samples under load (above half the max clock;
        all samples if none is), the max clock, and every throttle reason active in one of
        those samples.  Malformed lines are skipped."""
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smmax=float(parts[2]), hw=parts[5], hwt=parts[6],
                                 swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [r for r in rows if r["sm"] > 0.5 * r["smmax"]] or rows
        reasons = set()
        for r in busy:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in busy), "sm_max_mhz": busy[0]["smmax"],
                "reasons": sorted(reasons), "samples": len(busy)}


# ----------------------------------------------------------------------------- work units
def algorithmic(w: I.Workload, n_rep: int, fused: bool = False):
    """Algorithmic bytes (HBM) or flops per call for one step.  Fused: the dispatch call
    only reads idx and writes perm and src; the FFN reads the token rows itself."""
    T, E, k, d, F, A = w.T, w.E, w.k, w.d, w.F, w.A
    return {
        # top-k reads the logits and writes idx and gate; the histogram and the plan
        # (fused into the same launch) add only E-sized traffic
        "moe_route_plan": ("GB/s", T * E * 4 + A * 8),
        "moe_prefetch_replicas": ("GB/s", 2 * n_rep * 3 * d * F * 2),
        "moe_dispatch": ("GB/s", 12 * A if fused else T * d * 2 + A * d * 2 + 12 * A),
        "moe_grouped_ffn": ("TFLOP/s", 6 * A * d * F),
        "moe_combine": ("GB/s", A * d * 2 + T * d * 2 + 8 * A),
    }


CALLS = ["moe_route_plan", "moe_prefetch_replicas", "moe_dispatch", "moe_grouped_ffn",
         "moe_combine"]


def cudart():
    """The CUDA runtime already loaded by torch (for event-record graph nodes)."""
    import glob
    cands = ["libcudart.so.12", "libcudart.so"]
    base = os.path.join(os.path.dirname(torch.__file__), os.pardir, "nvidia", "cuda_runtime", "lib")
    cands += sorted(glob.glob(os.path.join(base, "libcudart.so*")))
    for c in cands:
        try:
            lib = ctypes.CDLL(c)
            lib.cudaEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
            lib.cudaEventRecordWithFlags.restype = ctypes.c_int
            return lib
        except (OSError, AttributeError):
            continue
    raise RuntimeError("CUDA runtime library not found")


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- our arm
def run_ours(args, w: I.Workload, world, rank, local):
    import load_balanced_dispatch_warp_b200 as M

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    logits_h = I.make_logits(w).pin_memory()
    x_h = I.make_x(w).pin_memory()
    logits = logits_h.to(device)
    x = x_h.to(device)
    W1, W3, W2 = I.make_weights(w, device=device)
    if args.ffn_tile is not None:
        M.set_ffn_tile_mode(args.ffn_tile)
    ffn_tile = int(M.lib().moe_ffn_tile_mode())
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F, device=device, fused=args.fused)
    # the per-call table: the forward's calls one after the other (event nodes between them)
    steps = [lambda: L.route_plan(logits), lambda: L.prefetch(W1, W3, W2),
             lambda: L.dispatch(x), lambda: L.expert_ffn(W1, W3, W2), lambda: L.combine()]

    for _ in range(max(args.warmup, 1)):
        L.forward(logits, x, W1, W3, W2)
    torch.cuda.synchronize()
    if int(L.err.item()) != 0:
        raise RuntimeError(f"device error word {int(L.err.item())} after warm-up")
    n_rep = int(L.plan_field("replica_list")[0].item())

    # device-timed region: K steps, events between the calls on the launching stream.
    # The K steps are captured once into a CUDA graph (no host launch gaps) and replayed.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(steps) + 1)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)

    for e in [start, end] + [x for row in ev for x in row]:
        e.record(stream)  # create the CUDA events before any capture
    torch.cuda.synchronize()

    def timed_steps(st, rec):
        rec(start, st)
        for s in range(args.steps):
            e = ev[s]
            rec(e[0], st)
            for i, f in enumerate(steps):
                f()
                rec(e[i + 1], st)
        rec(end, st)

    # Two captures of the same K steps: a clean one (the timed headline) and one with an
    # event-record node between consecutive calls (the per-call table, replayed right
    # after, also K steps between barriers).
    graph = graph_ev = None
    if not args.eager:
        rt = cudart()

        def rec_node(event, st):  # an event-record node inside the graph
            rc = rt.cudaEventRecordWithFlags(ctypes.c_void_p(event.cuda_event),
                                             ctypes.c_void_p(st.cuda_stream), 1)
            if rc != 0:
                raise RuntimeError(f"cudaEventRecordWithFlags failed ({rc})")

        def capture(with_events):
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(device)
            cap.wait_stream(stream)
            torch.cuda.synchronize()
            with torch.cuda.stream(cap):
                g.capture_begin()
                if with_events:
                    timed_steps(cap, rec_node)
                else:  # the timed headline: the layer's forward as a user calls it
                    for _ in range(args.steps):
                        L.forward(logits, x, W1, W3, W2)
                g.capture_end()
            torch.cuda.synchronize()
            g.replay()  # one untimed replay (warm instantiation)
            torch.cuda.synchronize()
            return g
        graph = capture(False)
        graph_ev = capture(True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark_start()
    if graph is not None:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        elapsed_ms = t0.elapsed_time(t1)
        graph_ev.replay()  # instrumented replay: per-call intervals
    else:
        timed_steps(stream, lambda e, st: e.record(st))
        torch.cuda.synchronize()
        elapsed_ms = start.elapsed_time(end)
    torch.cuda.synchronize()
    barrier(world)
    clocks.mark_end()
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(elapsed_ms, world, device)
    if int(L.err.item()) != 0:
        raise RuntimeError(f"device error word {int(L.err.item())} in the timed region")
    del graph, graph_ev
    per_call_ms = {c: sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps)) / args.steps
                   for i, c in enumerate(CALLS)}

    # end to end through the public API: every step copies its logits and tokens from
    # pinned host memory and its output back; HostPipeline overlaps those copies with the
    # neighbouring steps' compute (two device slots, three streams).
    from load_balanced_dispatch_warp_b200.pipeline import HostPipeline
    pipe = HostPipeline(L, W1, W3, W2)
    outs_h = [torch.empty(w.T, w.d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    batches = [(logits_h, x_h)] * args.steps
    pipe.run(batches[:2], outs_h)  # warm the streams and events
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    pipe.s_comp.wait_stream(pipe.s_in)
    pipe.run(batches, [outs_h[i % 2] for i in range(args.steps)])
    e1.record(pipe.s_out)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    if int(L.err.item()) != 0:
        raise RuntimeError(f"device error word {int(L.err.item())} in the end-to-end run")

    units = algorithmic(w, n_rep, args.fused)
    peaks, peak_src = load_peaks()
    calls = {}
    for c in CALLS:
        unit, work = units[c]
        ms = per_call_ms[c]
        rec = {"us": round(ms * 1e3, 2)}
        if work is not None and ms > 0:
            if unit == "TFLOP/s":
                ach = work / (ms * 1e-3) / 1e12
                peak = peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
            else:
                ach = work / (ms * 1e-3) / 1e9
                peak = peaks["hbm_gbs"]
            rec.update({unit.replace("/", "_per_"): round(ach, 1), "frac": round(ach / peak, 3)})
        calls[c] = rec
    ffn_ms = per_call_ms["moe_grouped_ffn"]
    ffn_flops = units["moe_grouped_ffn"][1]
    peak_t = peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
    achieved = ffn_flops / (ffn_ms * 1e-3) / 1e12
    tkey = f"{w.name}:{ffn_tile}:{sources_hash()}"
    roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak_t, "unit": "TFLOP/s",
                "frac": round(achieved / peak_t, 3), "traffic": TRAFFIC.get(tkey),
                "kernel": "moe_grouped_ffn (gate-up and down tcgen05 GEMMs)",
                "peak_source": f"{peak_src} sustained bf16 GEMM",
                "work_per_launch": f"6*A*d*F = {ffn_flops:.4g} flop (A=T*k={w.A})"}

    value = w.T * args.steps * world / (elapsed_ms * 1e-3)
    e2e_value = w.T * args.steps * world / (e2e_ms * 1e-3)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(elapsed_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16+fp16 (gate/up GEMM bf16, down GEMM fp16, fp32 accumulate; routing fp32)",
        "data": "synthetic (seeded; N(0,1) logits + per-expert bias, N(0,1) tokens, N(0,1/d) weights)",
        "config": {"workload": w.name, "T": w.T, "E": w.E, "k": w.k, "R": w.R, "S": w.S, "d": w.d,
                   "F": w.F, "maxvio": round(float(L.maxvio.item()), 4), "replicas": n_rep,
                   # makespan proxy: rows of the busiest rank / C, with the plan and with
                   # every expert at its home rank
                   "max_rank_rows_over_C": 1.0,
                   "home_only_max_rank_rows_over_C": round(1.0 + float(L.maxvio.item()), 4),
                   "parallelism": f"replicas x{world} (ranks simulated in one GPU's HBM)",
                   "dispatch": ("fused: placement only, GEMM 1 gathers x[src[row]]" if args.fused
                                else "row copy into recv, GEMM 1 reads recv"),
                   "ffn_tile": ("256-row tiles on 2-CTA clusters (tcgen05 cta_group::2)"
                                if ffn_tile == 1 and not args.fused
                                else "128-row tiles, one CTA each (tcgen05 cta_group::1)"),
                   "ffn_pair_clusters": M.ffn_pair_clusters() if ffn_tile == 1 else None,
                   "l2": "step working set (weights, pool, activations) far above the 126 MB L2",
                   "launch": "eager, one stream, calls in order" if args.eager else
                             "K forward steps (MoELayer.forward: routing/histogram/plan fused in "
                             "one launch, then prefetch, dispatch, FFN, combine) captured in one "
                             "CUDA graph, replayed once; per-call intervals from a second replay "
                             "with event nodes between the calls"},
        "clocks": clk,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT,
                "h2d_bytes_per_step": w.T * w.E * 4 + w.T * w.d * 2,
                "d2h_bytes_per_step": w.T * w.d * 2},
        "gpu_launches": L.kernels_per_forward() * args.steps,
        "roofline": roofline,
        "calls": calls,
    }
    if args.backward:
        res["train_step"] = time_training_step(args, w, L, logits, x, W1, W3, W2, world, device, peaks)
    return res


BWD_CALLS = ["moe_combine_backward", "moe_grouped_ffn_backward", "moe_dispatch_backward",
             "moe_topk_backward"]


def time_training_step(args, w: I.Workload, L, logits, x, W1, W3, W2, world, device, peaks):
    """Forward + backward of the layer (dout seeded N(0,1) bf16), K steps in one CUDA graph
    after warm-up; per-call backward intervals from a replay with event nodes between the
    calls.  The grouped-FFN backward does 16*A*d*F flops: dH (2AdF), the gate/up GEMM re-run
    (4AdF), dX rows (4AdF), dW2 (2AdF), dW1 and dW3 (4AdF)."""
    g = torch.Generator().manual_seed(41)
    dout = torch.randn(w.T, w.d, generator=g).to(torch.bfloat16).to(device)
    for _ in range(max(args.warmup, 1)):
        L.forward(logits, x, W1, W3, W2)
        L.backward(dout, W1, W3, W2)
    torch.cuda.synchronize()
    if int(L.err.item()) != 0:
        raise RuntimeError(f"device error word {int(L.err.item())} after the backward warm-up")
    import load_balanced_dispatch_warp_b200 as M
    b = L._bwd
    bsteps = [lambda: M.moe_combine_backward(dout, L.y, L.perm, L.gate, b["dy"], b["dgate"], L.err),
              lambda: M.moe_grouped_ffn_backward(L.recv, b["dy"], L.h, L.plan, W1, W3, W2, L.T, L.k, L.R,
                                                 L.S, b["dx_rows"], b["dW1"], b["dW3"], b["dW2"],
                                                 b["workspace"], L.err),
              lambda: M.moe_dispatch_backward(b["dx_rows"], L.perm, b["dx"], L.err),
              lambda: M.moe_topk_backward(L.gate, b["dgate"], L.idx, L.E, b["dlogits"], L.err)]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(bsteps) + 1)] for _ in range(args.steps)]
    for row in ev:
        for e in row:
            e.record()
    torch.cuda.synchronize()
    rt = cudart()

    def rec_node(event, st):
        rc = rt.cudaEventRecordWithFlags(ctypes.c_void_p(event.cuda_event), ctypes.c_void_p(st.cuda_stream), 1)
        if rc != 0:
            raise RuntimeError(f"cudaEventRecordWithFlags failed ({rc})")

    def capture(with_events):
        gr = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device)
        cap.wait_stream(torch.cuda.current_stream(device))
        torch.cuda.synchronize()
        with torch.cuda.stream(cap):
            gr.capture_begin()
            for st in range(args.steps):
                L.forward(logits, x, W1, W3, W2)
                if with_events:
                    rec_node(ev[st][0], cap)
                for i, f in enumerate(bsteps):
                    f()
                    if with_events:
                        rec_node(ev[st][i + 1], cap)
            gr.capture_end()
        torch.cuda.synchronize()
        gr.replay()
        torch.cuda.synchronize()
        return gr

    clean = capture(False)
    inst = capture(True)
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream(device)
    t0.record(stream)
    clean.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world, device)
    inst.replay()
    torch.cuda.synchronize()
    if int(L.err.item()) != 0:
        raise RuntimeError(f"device error word {int(L.err.item())} in the timed training steps")
    del clean, inst
    per = {c: sum(ev[st][i].elapsed_time(ev[st][i + 1]) for st in range(args.steps)) / args.steps
           for i, c in enumerate(BWD_CALLS)}
    A, d, F = w.A, w.d, w.F
    ffn_flops = 16 * A * d * F
    peak_t = peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
    calls = {c: {"us": round(v * 1e3, 2)} for c, v in per.items()}
    t_ffn = per["moe_grouped_ffn_backward"] * 1e-3
    calls["moe_grouped_ffn_backward"].update(
        {"TFLOP_per_s": round(ffn_flops / t_ffn / 1e12, 1), "frac": round(ffn_flops / t_ffn / 1e12 / peak_t, 3),
         "work": f"16*A*d*F = {ffn_flops:.4g} flop"})
    return {"value": round(w.T * args.steps * world / (ms * 1e-3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms / args.steps, 4),
            "what": "forward + backward (dx, dlogits, dW1, dW3, dW2) per step, K steps in one CUDA graph",
            "backward_calls": calls}


# ----------------------------------------------------------------------------- oracle
def oracle_sample_tokens(w: I.Workload) -> int:
    """Tokens per CPU-oracle step: a prefix of the batch, a multiple of R/gcd(k,R)."""
    import math
    unit = w.R // math.gcd(w.k, w.R)
    target = max(unit, int(3.0e10 / (6 * w.k * w.d * w.F)))  # about 30 GFLOP of fp64 FFN work
    target = min(target, w.T)
    return max(unit, target // unit * unit)


def run_oracle_step(w: I.Workload, logits, x, weights64_fn, Ts: int):
    from oracle import moe_oracle as O
    lg = logits[:Ts]
    xs = x[:Ts]
    idx, gate, err = O.topk_route(lg, w.k)
    h = O.expert_histogram(idx, w.E, w.R)
    p = O.plan_balanced(h["counts"], Ts, w.k, w.E, w.R, w.S)
    perm, src = O.permute(idx, p, w.E, w.R)
    recv = O.dispatch(xs, src)
    y = np.zeros((recv.shape[0], w.d))
    for gl in p["groups"]:
        for (r0, n, e, ref) in gl:
            w1, w3, w2 = weights64_fn(e)  # a replica slot holds these weights bitwise
            y[r0:r0 + n] = O.expert_ffn(recv[r0:r0 + n], w1, w3, w2)
    return O.combine(y, perm, gate)


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_inputs(w: I.Workload):
    import collections
    logits = I.make_logits(w).numpy()
    x = I.make_x(w).double().numpy()
    cache = collections.OrderedDict()  # fp64 copies of recently used experts (bounded)
    budget = max(1, int(8e9 // (3 * w.d * w.F * 8)))
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    W = I.make_weights(w, device=dev)

    def weights64(e):
        if e in cache:
            cache.move_to_end(e)
        else:
            cache[e] = tuple(t[e].to("cpu", torch.float64).numpy() for t in W)
            while len(cache) > budget:
                cache.popitem(last=False)
        return cache[e]
    return logits, x, weights64


def measure_oracle(w: I.Workload, steps: int, warmup: int, budget_s: float | None = None):
    logits, x, weights64 = oracle_inputs(w)
    Ts = oracle_sample_tokens(w)
    for _ in range(warmup):
        run_oracle_step(w, logits, x, weights64, Ts)
    t0 = time.perf_counter()
    n = 0
    for _ in range(steps):
        run_oracle_step(w, logits, x, weights64, Ts)
        n += 1
        if budget_s is not None and time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return Ts * n / dt, Ts, n, dt


def run_reference(args, w):
    world, rank, local = dist_env()
    if rank != 0:
        return None
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    value, Ts, n, dt = measure_oracle(w, args.steps, args.warmup, budget_s=120.0)
    cores = cpu_threads()
    sample = (f"first {Ts} of {w.T} tokens through the whole oracle layer per step, {n} of "
              f"{args.steps} steps (120 s budget)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 1,
        "steps": n, "warmup": args.warmup, "ms_per_step": round(dt / n * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "T": w.T, "E": w.E, "k": w.k, "R": w.R, "S": w.S, "d": w.d,
                   "F": w.F},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="near_balanced", choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch the timed steps eagerly")
    ap.add_argument("--backward", action="store_true",
                    help="also time the training step (forward + backward) and the backward calls")
    ap.add_argument("--fused", action="store_true",
                    help="fused dispatch: placement only, GEMM 1 gathers the token rows")
    ap.add_argument("--ffn-tile", type=int, default=None, choices=[0, 1],
                    help="grouped-FFN tiling: 0 = 128-row tiles, one CTA each; 1 = 256-row "
                         "tiles on 2-CTA clusters (default: the library's)")
    args = ap.parse_args()
    w = I.WORKLOADS[args.config]

    if args.impl == "reference":
        res = run_reference(args, w)
        if res is not None:
            print(json.dumps(res, sort_keys=True), flush=True)
        return

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    res = run_ours(args, w, world, rank, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        value, Ts, n, dt = measure_oracle(w, steps=1000, warmup=1, budget_s=15.0)
        res["cpu_baseline"] = {"value": round(value, 3), "unit": UNIT, "cores": cpu_threads(),
                               "kind": "oracle",
                               "sample": f"first {Ts} of {w.T} tokens through the whole oracle "
                                         f"layer, {n} passes in {dt:.1f} s"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res, sort_keys=True), flush=True)


if __name__ == "__main__":
    main()
