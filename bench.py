"""Throughput of the MoE-layer hot path on B200: one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one pass of the whole path (top-k, histogram/maxvio, balanced plan, replica
prefetch, dispatch, grouped SwiGLU FFN, combine) over one batch of seeded synthetic
inputs already resident in HBM.  The default workload is the largest single-GPU one, the
DeepSeek-V3-shaped hotspot layer (16384 tokens, 256 experts, top-8, 32 simulated ranks,
4 slots, d=7168, F=2048, ~90% of assignments on 26 hot experts).  At one GPU the line
also carries the stand-alone top-k against the copy floor of a launch of its size and the
Qwen-shaped maxvio sweep (tokens/s vs maxvio), each point with its own clock record.
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

# DRAM bytes (read + write) per call of the dominant call (both grouped-FFN kernels),
# dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of the two FFN kernels
# (`ncu --set full --clock-control none -k regex:ffn_kernel ...` on the named workload),
# keyed by workload, tile mode and kernel-sources hash: a kernel edit changes the hash,
# and the line then reports null (with the reason) until the counters are taken again.
TRAFFIC = {"deepseek:0:f6968ffe57135168": 22115675136 + 533353216 + 8993779968 + 1833654016}
TRAFFIC_NOTE = {"deepseek:0:f6968ffe57135168":
                "ncu dram__bytes_read.sum + dram__bytes_write.sum of the gate-up and down "
                "kernels of one full DeepSeek call (bench.py --only ffn --config deepseek)"}


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
def algorithmic(w: I.Workload, n_rep: int, fused: bool = False, fused_combine: bool = False):
    """Algorithmic bytes (HBM) or flops per call for one step.  Fused: the dispatch call
    only reads idx and writes perm and src; the FFN reads the token rows itself.  Fused
    combine: the FFN call also does the combine (its rate is still quoted on 6*A*d*F), the
    combine call does nothing."""
    T, E, k, d, F, A = w.T, w.E, w.k, w.d, w.F, w.A
    if fused_combine:
        return {
            "moe_route_plan": ("GB/s", T * E * 4 + A * 8),
            "moe_prefetch_replicas": ("GB/s", 2 * n_rep * 3 * d * F * 2),
            "moe_dispatch": ("GB/s", T * d * 2 + A * d * 2 + 12 * A),
            "moe_grouped_ffn": ("TFLOP/s", 6 * A * d * F),
            "moe_combine": ("GB/s", None),
        }
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
def ffn_peak(clk: dict, peaks: dict, peak_src: str):
    """The bf16 dense peak that matches the clocks the FFN ran at: the burst figure (a
    GEMM timed alone, SM clock at max) when the median SM clock under load sat within 3%
    of its max and the power cap never engaged, the sustained figure (seconds-long GEMM
    under the 1 kW cap) otherwise."""
    smmax = clk.get("sm_max_mhz") or peaks.get("sm_max_mhz") or 1965.0
    sm = clk.get("sm_mhz")
    burst = (sm is not None and sm >= 0.97 * smmax
             and "sw_power_cap" not in clk.get("reasons", []))
    if burst or not peaks.get("bf16_tflops_sustained"):
        return peaks["bf16_tflops"], f"{peak_src} burst bf16 GEMM (SM clock at max, no power cap)"
    return (peaks["bf16_tflops_sustained"],
            f"{peak_src} sustained bf16 GEMM (SM clock below max or power cap active)")


def rec_node_fn():
    """An event-record node inside a graph being captured (PyTorch's Event.record does not
    create one during capture)."""
    rt = cudart()

    def rec_node(event, st):
        rc = rt.cudaEventRecordWithFlags(ctypes.c_void_p(event.cuda_event),
                                         ctypes.c_void_p(st.cuda_stream), 1)
        if rc != 0:
            raise RuntimeError(f"cudaEventRecordWithFlags failed ({rc})")
    return rec_node


def measure_layer(args, w: I.Workload, world, device, steps: int, e2e: bool):
    """K forward steps of one workload: the clean graph (the timed value), the instrumented
    graph (per-call intervals), the clock record over both, and optionally the end-to-end
    run through HostPipeline.  Returns a dict of raw measurements and the layer."""
    import load_balanced_dispatch_warp_b200 as M

    stream = torch.cuda.current_stream(device)
    logits_h = I.make_logits(w).pin_memory()
    x_h = I.make_x(w).pin_memory()
    logits = logits_h.to(device)
    x = x_h.to(device)
    W1, W3, W2 = I.make_weights(w, device=device)
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F, device=device, fused=args.fused,
                   fused_combine=args.fused_combine)
    # the per-call table: the forward's calls one after the other (event nodes between them)
    calls = [lambda: L.route_plan(logits), lambda: L.prefetch(W1, W3, W2),
             lambda: L.dispatch(x), lambda: L.expert_ffn(W1, W3, W2), lambda: L.combine()]

    for _ in range(max(args.warmup, 1)):
        L.forward(logits, x, W1, W3, W2)
    torch.cuda.synchronize()
    if int(L.err.item()) != 0:
        raise RuntimeError(f"{w.name}: device error word {int(L.err.item())} after warm-up")
    n_rep = int(L.plan_field("replica_list")[0].item())

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
    for e in [x for row in ev for x in row]:
        e.record(stream)  # create the CUDA events before any capture
    torch.cuda.synchronize()

    # Two captures of the same K steps: a clean one (the timed headline: the layer's forward
    # as a user calls it) and one with an event-record node between consecutive calls.
    graph = graph_ev = None
    if not args.eager:
        rec_node = rec_node_fn()

        def capture(with_events):
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(device)
            cap.wait_stream(stream)
            torch.cuda.synchronize()
            with torch.cuda.stream(cap):
                g.capture_begin()
                for s in range(steps):
                    if with_events:
                        rec_node(ev[s][0], cap)
                        for i, f in enumerate(calls):
                            f()
                            rec_node(ev[s][i + 1], cap)
                    else:
                        L.forward(logits, x, W1, W3, W2)
                g.capture_end()
            torch.cuda.synchronize()
            g.replay()  # one untimed replay (warm instantiation)
            torch.cuda.synchronize()
            return g
        graph = capture(False)
        graph_ev = capture(True)
    clocks = ClockSampler(device.index)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if graph is not None:
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        elapsed_ms = t0.elapsed_time(t1)
        graph_ev.replay()  # instrumented replay: per-call intervals
    else:
        t0.record(stream)
        for s in range(steps):
            ev[s][0].record(stream)
            for i, f in enumerate(calls):
                f()
                ev[s][i + 1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        elapsed_ms = t0.elapsed_time(t1)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(elapsed_ms, world, device)
    if int(L.err.item()) != 0:
        raise RuntimeError(f"{w.name}: device error word {int(L.err.item())} in the timed region")
    del graph, graph_ev
    per_call_ms = {c: sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)) / steps
                   for i, c in enumerate(CALLS)}
    out = dict(layer=L, n_rep=n_rep, elapsed_ms=elapsed_ms, per_call_ms=per_call_ms, clocks=clk,
               maxvio=float(L.maxvio.item()))

    if e2e:
        # end to end through the public API: every step copies its logits and tokens from
        # pinned host memory and its output back; HostPipeline overlaps those copies with
        # the neighbouring steps' compute (two device slots, three streams).
        from load_balanced_dispatch_warp_b200.pipeline import HostPipeline
        pipe = HostPipeline(L, W1, W3, W2)
        outs_h = [torch.empty(w.T, w.d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        batches = [(logits_h, x_h)] * steps
        pipe.run(batches[:2], outs_h)  # warm the streams and events
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(pipe.s_in)
        pipe.s_comp.wait_stream(pipe.s_in)
        pipe.run(batches, [outs_h[i % 2] for i in range(steps)])
        e1.record(pipe.s_out)
        torch.cuda.synchronize()
        barrier(world)
        out["e2e_ms"] = max_over_ranks(e0.elapsed_time(e1), world, device)
        if int(L.err.item()) != 0:
            raise RuntimeError(f"{w.name}: device error word {int(L.err.item())} in the e2e run")
    out["weights"] = (W1, W3, W2)
    out["inputs"] = (logits, x)
    return out


def call_table(w: I.Workload, m: dict, peaks: dict, fused: bool, tflops_peak: float,
               fused_combine: bool = False):
    """Per-call rates: algorithmic work over the in-graph interval, as a fraction of the
    measured copy peak (HBM-bound calls) or of the clock-matched bf16 peak (the FFN)."""
    units = algorithmic(w, m["n_rep"], fused, fused_combine)
    calls = {}
    for c in CALLS:
        unit, work = units[c]
        ms = m["per_call_ms"][c]
        rec = {"us": round(ms * 1e3, 2)}
        if work is not None and ms > 0:
            if unit == "TFLOP/s":
                ach, peak = work / (ms * 1e-3) / 1e12, tflops_peak
            else:
                ach, peak = work / (ms * 1e-3) / 1e9, peaks["hbm_gbs"]
            rec.update({unit.replace("/", "_per_"): round(ach, 1), "frac": round(ach / peak, 3)})
        calls[c] = rec
    return calls


def topk_floor(w: I.Workload, device, reps: int = 200, copies: int = 16):
    """Stand-alone moe_topk against the copy floor of a launch of its size.  Both run on
    `copies` rotating input buffers (copies x T*E*4 bytes, far above the 126 MB L2) so that
    each launch reads HBM, `reps` launches captured in one CUDA graph and replayed between
    CUDA events.  The
    floor is a device copy (torch copy_) whose read + write bytes equal the top-k's
    algorithmic bytes (T*E*4 + A*8), and a copy of exactly T*E*4 bytes for reference."""
    import load_balanced_dispatch_warp_b200 as M
    stream = torch.cuda.current_stream(device)
    g = torch.Generator(device=device).manual_seed(5)
    srcs = [torch.randn(w.T, w.E, generator=g, device=device) for _ in range(copies)]
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=device)
    gate = torch.empty(w.T, w.k, dtype=torch.float32, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)

    def timed(fn):
        # the reps launches captured in one CUDA graph: a launch this short is faster than
        # the host can issue it one call at a time (an empty kernel with this grid, issued
        # eagerly through the binding, measured the same ~13.5 us as the top-k), so only a
        # graph replay shows the device time
        for i in range(copies):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            g.capture_begin()
            for r in range(reps):
                fn(r % copies)
            g.capture_end()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / reps * 1e3  # us per launch

    topk_us = timed(lambda i: M.moe_topk(srcs[i], w.k, idx, gate, err))
    alg = w.T * w.E * 4 + w.A * 8
    half = [torch.empty(alg // 2 // 4, dtype=torch.float32, device=device) for _ in range(2 * copies)]
    copy_us = timed(lambda i: half[2 * i].copy_(half[2 * i + 1]))
    full = [torch.empty(w.T * w.E, dtype=torch.float32, device=device) for _ in range(2 * copies)]
    copy_full_us = timed(lambda i: full[2 * i].copy_(full[2 * i + 1]))
    if int(err.item()) != 0:
        raise RuntimeError("moe_topk set the error word on random logits")
    del srcs, half, full
    torch.cuda.empty_cache()
    topk_gbs = alg / (topk_us * 1e-6) / 1e9
    floor_gbs = (alg // 2 // 4 * 4 * 2) / (copy_us * 1e-6) / 1e9
    return {"us": round(topk_us, 2), "GB_per_s": round(topk_gbs, 1),
            "algorithmic_bytes": alg,
            "copy_floor_us": round(copy_us, 2), "copy_floor_GB_per_s": round(floor_gbs, 1),
            "frac_of_copy_floor": round(topk_gbs / floor_gbs, 3),
            "copy_of_logits_us": round(copy_full_us, 2),
            "what": f"moe_topk alone, {copies} rotating logits buffers, {reps} launches in one "
                    f"CUDA graph; floor = torch copy_ moving the same bytes (read + write), same "
                    f"rotation, same graph timing"}


def summarize(w: I.Workload, m: dict, peaks: dict, peak_src: str, fused: bool, steps: int,
              fused_combine: bool = False):
    """Compact record of one workload: tokens/s, the per-call table, the FFN against the
    clock-matched peak, and the FFN's duration in SM cycles at the median clock."""
    tpk, tpk_src = ffn_peak(m["clocks"], peaks, peak_src)
    calls = call_table(w, m, peaks, fused, tpk, fused_combine)
    ffn_us = m["per_call_ms"]["moe_grouped_ffn"] * 1e3
    sm = m["clocks"].get("sm_mhz")
    return {"value": round(w.T * steps / (m["elapsed_ms"] * 1e-3), 1),
            "ms_per_step": round(m["elapsed_ms"] / steps, 4), "maxvio": round(m["maxvio"], 4),
            "replicas": m["n_rep"], "calls": calls, "clocks": m["clocks"],
            "ffn_peak": tpk, "ffn_peak_source": tpk_src,
            "ffn_mcycles": round(ffn_us * sm / 1e6, 4) if sm else None}


def run_ours(args, w: I.Workload, world, rank, local):
    import load_balanced_dispatch_warp_b200 as M

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.ffn_tile is not None:
        M.set_ffn_tile_mode(args.ffn_tile)
    ffn_tile = int(M.lib().moe_ffn_tile_mode())
    peaks, peak_src = load_peaks()

    m = measure_layer(args, w, world, device, args.steps, e2e=True)
    L = m["layer"]
    head = summarize(w, m, peaks, peak_src, args.fused, args.steps, args.fused_combine)
    units = algorithmic(w, m["n_rep"], args.fused, args.fused_combine)
    ffn_ms = m["per_call_ms"]["moe_grouped_ffn"]
    ffn_flops = units["moe_grouped_ffn"][1]
    achieved = ffn_flops / (ffn_ms * 1e-3) / 1e12
    tkey = f"{w.name}:{ffn_tile}:{sources_hash()}"
    traffic = TRAFFIC.get(tkey)
    roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": head["ffn_peak"],
                "unit": "TFLOP/s", "frac": round(achieved / head["ffn_peak"], 3),
                "traffic": traffic,
                "traffic_note": (TRAFFIC_NOTE.get(tkey) if traffic is not None else
                                 "null: no ncu DRAM capture of this workload at these kernel "
                                 f"sources (key {tkey})"),
                "kernel": "moe_grouped_ffn (gate-up and down tcgen05 GEMMs)",
                "peak_source": head["ffn_peak_source"],
                "ffn_mcycles_at_median_sm_clock": head["ffn_mcycles"],
                "work_per_launch": f"6*A*d*F = {ffn_flops:.4g} flop (A=T*k={w.A})"}

    value = w.T * args.steps * world / (m["elapsed_ms"] * 1e-3)
    e2e_value = w.T * args.steps * world / (m["e2e_ms"] * 1e-3)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(m["elapsed_ms"] / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16+fp16 (gate/up GEMM bf16, down GEMM fp16, fp32 accumulate; routing fp32)",
        "data": "synthetic (seeded; N(0,1) logits + per-expert bias, N(0,1) tokens, N(0,1/d) weights)",
        "config": {"workload": w.name, "T": w.T, "E": w.E, "k": w.k, "R": w.R, "S": w.S, "d": w.d,
                   "F": w.F, "maxvio": round(m["maxvio"], 4), "replicas": m["n_rep"],
                   # makespan proxy: rows of the busiest rank / C, with the plan and with
                   # every expert at its home rank
                   "max_rank_rows_over_C": 1.0,
                   "home_only_max_rank_rows_over_C": round(1.0 + m["maxvio"], 4),
                   "parallelism": f"replicas x{world} (ranks simulated in one GPU's HBM)",
                   "dispatch": ("fused: placement only, GEMM 1 gathers x[src[row]]" if args.fused
                                else "row copy into recv, GEMM 1 reads recv"),
                   "combine": ("fused into GEMM 2's epilogue (fp32 atomics, then bf16)"
                               if args.fused_combine else "separate gather kernel, j-ordered"),
                   "ffn_tile": ("256-row tiles on 2-CTA clusters (tcgen05 cta_group::2)"
                                if ffn_tile == 1 and not args.fused
                                else "128-row tiles, one CTA each (tcgen05 cta_group::1)"),
                   "ffn_pair_clusters": M.ffn_pair_clusters() if ffn_tile == 1 else None,
                   "l2": "inputs larger than L2: the step's working set (weights, pool, "
                         "activations) is far above the 126 MB L2, no flush inserted",
                   "launch": "eager, one stream, calls in order" if args.eager else
                             "K forward steps (MoELayer.forward: routing/histogram/plan fused in "
                             "one launch, then prefetch, dispatch, FFN, combine) captured in one "
                             "CUDA graph, replayed once; per-call intervals from a second replay "
                             "with event nodes between the calls"},
        "clocks": m["clocks"],
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT,
                "h2d_bytes_per_step": w.T * w.E * 4 + w.T * w.d * 2,
                "d2h_bytes_per_step": w.T * w.d * 2},
        "gpu_launches": L.kernels_per_forward() * args.steps,
        "roofline": roofline,
        "calls": head["calls"],
    }
    if args.backward:
        W1, W3, W2 = m["weights"]
        logits, x = m["inputs"]
        res["train_step"] = time_training_step(args, w, L, logits, x, W1, W3, W2, world, device,
                                               peaks, head["ffn_peak"])
    del m, L
    torch.cuda.empty_cache()
    if world == 1 and not args.no_extras:
        res["topk_standalone"] = topk_floor(w, device)
        sweep = {}
        for name in SWEEP:
            ws = I.WORKLOADS[name]
            ms = measure_layer(args, ws, world, device, args.sweep_steps, e2e=False)
            sweep[name] = summarize(ws, ms, peaks, peak_src, args.fused, args.sweep_steps,
                                    args.fused_combine)
            del ms
            torch.cuda.empty_cache()
        res["maxvio_sweep"] = {"workloads": sweep, "steps": args.sweep_steps,
                               "what": "Qwen3-30B-A3B-shaped layer (T=8192, E=128, k=8, R=16, "
                                       "S=8, d=2048, F=768) at maxvio 0.2 / 1 / 5 / 15 "
                                       "(15 = the largest this R allows, standing in for 20)"}
    return res


def run_ep(args, w: I.Workload, world, rank, local):
    """Expert parallelism across GPUs (``--ep``).  N = 1: the workload's R ranks run in one
    process on this GPU (each rank's buffers separate allocations, the pointer tables
    standing in for peer mappings, the all-gather a device copy); the timed K steps are
    captured in one CUDA graph, and a second capture with event nodes between the stages
    gives each stage's time.  N > 1: one rank per GPU (R = N) over NCCL with the peers'
    buffers mapped through CUDA IPC, the workload's T tokens split over the ranks
    (strong scaling), K eager steps between barriers, max over ranks."""
    import load_balanced_dispatch_warp_b200 as M
    from load_balanced_dispatch_warp_b200.ep import EPLayer, EPRank, LocalRanks, NcclComm

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream(device)
    W = w.R if world == 1 else world
    if w.E % W or w.T % W:
        raise SystemExit(f"--ep: {w.name} cannot be split over {W} ranks (E={w.E}, T={w.T})")
    B, Tl = w.E // W, w.T // W
    logits = I.make_logits(w).to(device)
    x = I.make_x(w).to(device)
    W1, W3, W2 = I.make_weights(w, device=device)

    def shard(t, u):
        return t[u * Tl:(u + 1) * Tl].contiguous()

    stages = None
    if world == 1:
        lr = LocalRanks([EPRank(u, W, Tl, w.E, w.k, w.S, W1[u * B:(u + 1) * B],
                                W3[u * B:(u + 1) * B], W2[u * B:(u + 1) * B]) for u in range(W)])
        stages = lr.stages([shard(logits, u) for u in range(W)], [shard(x, u) for u in range(W)])
        if args.backward:
            g = torch.Generator(device=device).manual_seed(41)
            dout = torch.randn(w.T, w.d, generator=g, device=device).to(torch.bfloat16)
            stages = stages + lr.backward_stages([shard(dout, u) for u in range(W)])
        ranks = lr.ranks

        def step():
            for _, f in stages:
                f()
    else:
        own = tuple(t[rank * B:(rank + 1) * B].contiguous() for t in (W1, W3, W2))
        del W1, W3, W2
        torch.cuda.empty_cache()
        layer = EPLayer(NcclComm(), Tl, w.E, w.k, w.S, *own, backward=args.backward)
        lg, xs = shard(logits, rank), shard(x, rank)
        ranks = [layer.rank]
        if args.backward:
            g = torch.Generator(device=device).manual_seed(41)
            dout_own = shard(torch.randn(w.T, w.d, generator=g, device=device).to(torch.bfloat16), rank)

        def step():
            layer.forward(lg, xs)
            if args.backward:
                layer.backward(dout_own)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    errs = [int(r.err.item()) for r in ranks]
    if any(errs):
        raise RuntimeError(f"{w.name}: device error words {errs} after warm-up")
    n_rep = int(ranks[0].plan[M.plan_layout(w.E, W, w.S).replica_list].item())
    steps = args.steps
    stage_ms = None
    if world == 1:
        rec_node = rec_node_fn()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
              for _ in range(steps)]
        for e in [e for row in ev for e in row]:
            e.record(stream)
        torch.cuda.synchronize()

        def capture(with_events):
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(device)
            cap.wait_stream(stream)
            torch.cuda.synchronize()
            with torch.cuda.stream(cap):
                g.capture_begin()
                for si in range(steps):
                    if with_events:
                        rec_node(ev[si][0], cap)
                    for i, (_, f) in enumerate(stages):
                        f()
                        if with_events:
                            rec_node(ev[si][i + 1], cap)
                g.capture_end()
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            return g
        graph, graph_ev = capture(False), capture(True)
    clocks = ClockSampler(device.index)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    if world == 1:
        graph.replay()
    else:
        for _ in range(steps):
            step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = t0.elapsed_time(t1)
    if world == 1:
        graph_ev.replay()
        torch.cuda.synchronize()
        stage_ms = {name: sum(ev[si][i].elapsed_time(ev[si][i + 1]) for si in range(steps)) / steps
                    for i, (name, _) in enumerate(stages)}
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(elapsed_ms, world, device)
    errs = [int(r.err.item()) for r in ranks]
    if any(errs):
        raise RuntimeError(f"{w.name}: device error words {errs} in the timed region")
    row_bytes = w.d * 2
    work = {"dispatch": (w.T + w.A) * row_bytes, "combine": (w.A + w.T) * row_bytes,
            "prefetch": 2 * n_rep * 3 * w.d * w.F * 2, "ffn": 6 * w.A * w.d * w.F,
            "bwd_ffn": 16 * w.A * w.d * w.F}
    ffn_peak_v, ffn_src = ffn_peak(clk, peaks, peak_src)
    res = {
        "metric": METRIC, "value": round(w.T * steps / (elapsed_ms * 1e-3), 1), "unit": UNIT,
        "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / steps, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16+fp16 (gate/up GEMM bf16, down GEMM fp16, fp32 accumulate; routing fp32)",
        "data": "synthetic (seeded; N(0,1) logits + per-expert bias, N(0,1) tokens, N(0,1/d) weights)",
        "config": {"workload": w.name, "T": w.T, "E": w.E, "k": w.k, "R": W, "S": w.S, "d": w.d,
                   "F": w.F, "tokens_per_rank": Tl, "replicas": n_rep,
                   "parallelism": (f"ep{W}: {W} ranks in one process on one GPU (local buffers "
                                   "through the pointer tables stand in for peer mappings)"
                                   if world == 1 else
                                   f"ep{W}: one rank per GPU, NCCL all-gather and barriers, "
                                   "peer buffers through CUDA IPC"),
                   "l2": "inputs larger than L2 (weights, pool, activations), no flush",
                   "launch": ("K steps of every rank's stages captured in one CUDA graph"
                              if world == 1 else "eager, K steps between barriers"),
                   "step": ("forward + backward (dx, dlogits, home experts' weight gradients "
                            "with the replicas' reduced home)" if args.backward else "forward")},
        "clocks": clk,
        "e2e": None,
        # per rank and step: error-word reset and top-k, send-vector reset and counts,
        # plan, prefetch, workspace reset, dispatch rank pass and row stores, group table,
        # GEMM 1, GEMM 2, combine
        "gpu_launches": 13 * len(ranks) * steps,
    }
    if stage_ms is not None:
        st = {}
        for name, ms in stage_ms.items():
            row = {"us": round(ms * 1e3, 2)}
            if name in ("dispatch", "combine", "prefetch") and ms > 0:
                gbs = work[name] / (ms * 1e-3) / 1e9
                row.update(GB_per_s=round(gbs, 1), frac=round(gbs / peaks["hbm_gbs"], 3))
            if name in ("ffn", "bwd_ffn") and ms > 0:
                tf = work[name] / (ms * 1e-3) / 1e12
                row.update(TFLOP_per_s=round(tf, 1), frac=round(tf / ffn_peak_v, 3),
                           peak_source=ffn_src)
            st[name] = row
        res["ep_stages"] = st
        res["roofline"] = {"bound": "tensor", "achieved": st["ffn"].get("TFLOP_per_s"),
                           "peak": ffn_peak_v, "unit": "TFLOP/s", "frac": st["ffn"].get("frac"),
                           "traffic": None, "kernel": "moe_ep_grouped_ffn, all ranks",
                           "peak_source": ffn_src}
    if world > 1:
        layer.close()
    return res


def run_only(args, w: I.Workload):
    """One call of the path on its own, `--steps` calls captured in one CUDA graph and timed
    between CUDA events after `--warmup` eager calls: the case for kernel-level counter
    captures (ncu), which must stay a few GB on the device.  Prints one JSON line with the per-call time and rate; it is not
    the benchmark line."""
    import load_balanced_dispatch_warp_b200 as M
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    peaks, _ = load_peaks()
    if args.ffn_tile is not None:
        M.set_ffn_tile_mode(args.ffn_tile)
    res = {"only": args.only, "workload": w.name, "steps": args.steps,
           "ffn_tile": int(M.lib().moe_ffn_tile_mode())}
    if args.only == "topk":
        res.update(topk_floor(w, device, reps=args.steps))
        print(json.dumps(res, sort_keys=True), flush=True)
        return
    stream = torch.cuda.current_stream(device)
    i32 = torch.int32
    logits = I.make_logits(w).to(device)
    x = I.make_x(w).to(device)
    lay = M.plan_layout(w.E, w.R, w.S)
    idx = torch.empty(w.T, w.k, dtype=i32, device=device)
    gate = torch.empty(w.T, w.k, dtype=torch.float32, device=device)
    counts = torch.empty(w.E, dtype=i32, device=device)
    loads = torch.empty(w.R, dtype=i32, device=device)
    mv = torch.empty(1, dtype=torch.float64, device=device)
    bal = torch.empty(1, dtype=torch.float64, device=device)
    plan = torch.empty(lay.words, dtype=i32, device=device)
    rpw = torch.empty(M.route_plan_workspace_words(w.E), dtype=i32, device=device)
    err = torch.zeros(1, dtype=i32, device=device)
    ws = torch.empty(max(1, M.dispatch_workspace_words(w.T, w.E)), dtype=i32, device=device)
    perm = torch.empty(w.T, w.k, dtype=i32, device=device)
    src = torch.empty(w.A, dtype=i32, device=device)
    recv = torch.empty(w.A, w.d, dtype=torch.bfloat16, device=device)

    def route():
        M.moe_route_plan(logits, w.k, w.R, w.S, idx, gate, counts, loads, mv, bal, plan, rpw, err)

    def dispatch():
        M.moe_dispatch(x, idx, plan, w.E, w.R, w.S, ws, recv, perm, src, err)

    route()
    dispatch()
    units = algorithmic(w, 0)
    if args.only == "route":
        fn, unit, work = route, *units["moe_route_plan"]
    elif args.only == "dispatch":
        fn, unit, work = dispatch, *units["moe_dispatch"]
    elif args.only == "combine":
        y = recv.clone()
        out = torch.empty(w.T, w.d, dtype=torch.bfloat16, device=device)
        fn, unit, work = (lambda: M.moe_combine(y, perm, gate, out, err)), *units["moe_combine"]
    elif args.only == "prefetch":
        W1, W3, W2 = I.make_weights(w, device=device)
        P = [torch.empty(w.R * w.S, *t.shape[1:], dtype=t.dtype, device=device) for t in (W1, W3, W2)]
        n_rep = int(plan[lay.replica_list].item())
        fn = lambda: M.moe_prefetch_replicas(plan, W1, W3, W2, w.R, w.S, *P, err)
        unit, work = algorithmic(w, n_rep)["moe_prefetch_replicas"]
    else:  # ffn
        W1, W3, W2 = I.make_weights(w, device=device)
        P = [torch.empty(w.R * w.S, *t.shape[1:], dtype=t.dtype, device=device) for t in (W1, W3, W2)]
        M.moe_prefetch_replicas(plan, W1, W3, W2, w.R, w.S, *P, err)
        h = torch.empty(w.A, w.F, dtype=torch.float16, device=device)
        y = torch.empty(w.A, w.d, dtype=torch.bfloat16, device=device)
        fn = lambda: M.moe_grouped_ffn(recv, plan, W1, W3, W2, *P, w.T, w.k, w.R, w.S, h, y, err)
        unit, work = units["moe_grouped_ffn"]
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    # the `--steps` calls captured in one CUDA graph (short calls are otherwise bound by the
    # host issuing them), replayed once untimed, then once between CUDA events
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        g.capture_begin()
        for _ in range(args.steps):
            fn()
        g.capture_end()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    del g
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    us = a.elapsed_time(b) / args.steps * 1e3
    rate = work / (us * 1e-6) / (1e12 if unit == "TFLOP/s" else 1e9)
    peak = peaks["bf16_tflops"] if unit == "TFLOP/s" else peaks["hbm_gbs"]
    res.update({"us": round(us, 2), unit.replace("/", "_per_"): round(rate, 1),
                "frac": round(rate / peak, 3),
                "peak": "burst bf16 GEMM" if unit == "TFLOP/s" else "copy"})
    print(json.dumps(res, sort_keys=True), flush=True)


# Qwen-shaped skew sweep carried beside the headline (tokens/s vs maxvio)
SWEEP = ["qwen_mv0.2", "qwen_mv1", "qwen_mv5", "qwen_mv15"]


BWD_CALLS = ["moe_combine_backward", "moe_grouped_ffn_backward", "moe_dispatch_backward",
             "moe_topk_backward"]


def time_training_step(args, w: I.Workload, L, logits, x, W1, W3, W2, world, device, peaks,
                       peak_t):
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
    rec_node = rec_node_fn()

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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="deepseek", choices=sorted(I.WORKLOADS))
    ap.add_argument("--sweep-steps", type=int, default=50,
                    help="steps per point of the Qwen-shaped maxvio sweep")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the stand-alone top-k floor and the maxvio sweep")
    ap.add_argument("--only", default=None,
                    choices=["topk", "route", "dispatch", "combine", "prefetch", "ffn"],
                    help="time one call alone (--steps launches after --warmup) and print its "
                         "rate instead of the benchmark line: the small case for counter captures")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch the timed steps eagerly")
    ap.add_argument("--backward", action="store_true",
                    help="also time the training step (forward + backward) and the backward calls")
    ap.add_argument("--fused", action="store_true",
                    help="fused dispatch: placement only, GEMM 1 gathers the token rows")
    ap.add_argument("--fused-combine", action="store_true",
                    help="fused combine: GEMM 2's epilogue adds the gate-weighted rows into an "
                         "fp32 output (atomics), no y buffer and no combine kernel")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism across GPUs: one rank per GPU (R = N) for N > 1; "
                         "at N = 1 the workload's R ranks in one process on this GPU")
    ap.add_argument("--ffn-tile", type=int, default=None, choices=[0, 1],
                    help="grouped-FFN tiling: 0 = 128-row tiles, one CTA each; 1 = 256-row "
                         "tiles on 2-CTA clusters (default: the library's)")
    args = ap.parse_args()
    w = I.WORKLOADS[args.config]

    if args.only is not None:
        run_only(args, w)
        return
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
    if args.ep:
        res = run_ep(args, w, world, rank, local)
    else:
        res = run_ours(args, w, world, rank, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.ep:
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
