"""bench.py's host-side bookkeeping on CPU: the clock record taken during the timed region
(which decides whether a run is kept: a hardware or thermal slowdown, or clocks stuck
low, rejects it) and the per-call work units of the roofline."""
import bench
from load_balanced_dispatch_warp_b200 import inputs as I

NOT, ACT = "Not Active", "Active"


def line(sm, smmax=1965, hw=NOT, hwt=NOT, swt=NOT, pcap=NOT, power=900.0):
    return f"0, {sm}, {smmax}, {power}, 0x0, {hw}, {hwt}, {swt}, {pcap}"


def test_median_over_loaded_samples_and_reasons():
    out = "\n".join([
        line(345),                         # idle before the timed work: not under load
        line(1800, pcap=ACT),
        line(1700, pcap=ACT),
        line(1900),
        "garbage, line",                   # skipped
        line(1750, hwt=ACT),
        line(120),                         # idle after
    ])
    rec = bench.ClockSampler.summarize(out)
    assert rec["samples"] == 4
    assert rec["sm_mhz"] == 1775.0         # median of 1700, 1750, 1800, 1900
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_all_idle_samples_are_used_and_a_lock_shows():
    # clocks held at 900 MHz during the work (a leftover lock) sit below half the max clock:
    # every sample counts, and the record shows the low median with no reason
    out = "\n".join(line(900) for _ in range(5))
    rec = bench.ClockSampler.summarize(out)
    assert rec["sm_mhz"] == 900.0 and rec["reasons"] == [] and rec["samples"] == 5


def test_every_slowdown_reason_is_named():
    out = "\n".join([line(1500, hw=ACT), line(1500, swt=ACT), line(1500, pcap=ACT)])
    assert bench.ClockSampler.summarize(out)["reasons"] == [
        "hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]


def test_no_samples():
    assert bench.ClockSampler.summarize("")["reasons"] == ["no samples"]
    assert bench.ClockSampler.summarize("a,b\n")["sm_mhz"] is None


def test_work_units_of_the_default_workload():
    """Per-call work at near_balanced, from the tensors each call must read and write."""
    w = I.WORKLOADS["near_balanced"]
    T, E, k, d, F = w.T, w.E, w.k, w.d, w.F
    A = T * k
    n_rep = 8
    u = bench.algorithmic(w, n_rep)
    assert set(u) == set(bench.CALLS)
    bf16 = 2
    logits, idx_gate = T * E * 4, T * k * (4 + 4)
    assert u["moe_route_plan"] == ("GB/s", logits + idx_gate)
    x_rows, recv_rows = T * d * bf16, A * d * bf16
    idx_read, perm_write, src_write = 4 * A, 4 * A, 4 * A
    assert u["moe_dispatch"] == ("GB/s", x_rows + recv_rows + idx_read + perm_write + src_write)
    y_rows, out_rows, perm_gate = A * d * bf16, T * d * bf16, A * (4 + 4)
    assert u["moe_combine"] == ("GB/s", y_rows + out_rows + perm_gate)
    # each replica slot copies three [F, d] / [d, F] 16-bit matrices: read + write
    assert u["moe_prefetch_replicas"] == ("GB/s", n_rep * 3 * (F * d * 2) * 2)
    # gate, up and down projections of every useful row: three d x F GEMMs, 2 flop per MAC
    assert u["moe_grouped_ffn"] == ("TFLOP/s", 3 * 2 * A * d * F)
    # fused dispatch: no row copy; the FFN reads the token rows itself
    assert bench.algorithmic(w, n_rep, fused=True)["moe_dispatch"] == ("GB/s", 12 * A)


def test_reference_arm_line_keeps_the_contract(monkeypatch):
    """`bench.py --impl reference` on the tiny workload (the oracle on this host's cores):
    the JSON line carries the keys the contract names, with this arm's metric and unit."""
    import argparse
    import json
    for var in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(var, raising=False)
    args = argparse.Namespace(steps=2, warmup=1)
    line = bench.run_reference(args, I.WORKLOADS["tiny"])
    json.dumps(line)  # serialisable as printed
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["n_gpus"] == 1 and line["steps"] >= 1 and line["warmup"] == 1
    assert line["config"]["workload"] == "tiny"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert cb["unit"] == bench.UNIT and isinstance(cb["sample"], str)
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == bench.UNIT
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert line["vs_baseline"] is None


def test_ffn_peak_follows_the_clock_record():
    """The FFN's roofline denominator matches the clocks it ran at: the burst GEMM peak
    when the median SM clock sat at max with no power cap, the sustained one otherwise."""
    peaks = {"bf16_tflops": 1702.2, "bf16_tflops_sustained": 1430.7, "sm_max_mhz": 1965.0}
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    low = {"sm_mhz": 1207.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.ffn_peak(at_max, peaks, "measured")[0] == 1702.2
    assert "burst" in bench.ffn_peak(at_max, peaks, "measured")[1]
    assert bench.ffn_peak(capped, peaks, "measured")[0] == 1430.7
    assert bench.ffn_peak(low, peaks, "measured")[0] == 1430.7
    assert "sustained" in bench.ffn_peak(low, peaks, "measured")[1]
    # a record without samples cannot show the burst conditions
    assert bench.ffn_peak({"sm_mhz": None, "reasons": ["no samples"]}, peaks, "measured")[0] == 1430.7
