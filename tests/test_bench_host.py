"""Host logic of bench.py that needs no GPU: the NVML clock sampler (against a
fake NVML module), the algorithmic byte and FLOP counts, and the rule that a
recorded ncu traffic figure is reported only while the kernel sources are the
captured ones."""
import json
import os
import sys
import time
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from routed_expert_ffn_sqrtsoftplus_b200 import synth  # noqa: E402


def _fake_nvml(clocks, reasons):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    state = {"i": 0}
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByIndex = lambda i: ("dev", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        state["i"] += 1
        return clocks[state["i"] % len(clocks)]

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons
    return m


def test_clock_sampler_with_fake_nvml(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965, 1800, 1700], 0x4 | 0x1))
    with bench.ClockSampler(0, period_s=0.005) as clk:
        time.sleep(0.1)
    s = clk.summary()
    assert s["samples"] > 3
    assert s["sm_max_mhz"] == 1965
    assert s["sm_mhz"] in (1700, 1800, 1965)
    # gpu_idle is never reported; sw_power_cap is
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_reports_slowdowns(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1200], 0x8 | 0x40))
    with bench.ClockSampler(0, period_s=0.005) as clk:
        time.sleep(0.05)
    assert clk.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_clock_sampler_without_nvml(monkeypatch):
    bad = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no NVML")

    bad.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", bad)
    with bench.ClockSampler(0) as clk:
        pass
    assert clk.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_mxfp4_expert_bytes_match_the_pages_figure():
    """The bench's MXFP4 byte count per routed expert (gate/up + down) equals the
    18,800,640 B per expert that the pages' 18.8 MB figure rounds."""
    wl = synth.WORKLOADS["flash_mxfp4_decode"]
    one = bench.algorithmic(wl, np.array([[5]]), 1)
    k_gu, _ = one["kern"]["gemm_gateup_mx"]
    k_dn, _ = one["kern"]["gemm_down_mx"]
    rows = 1 * wl.k
    act_gu = rows * (wl.H + wl.I)
    act_dn = rows * wl.I + rows * wl.H * 4
    assert (k_gu - act_gu) + (k_dn - act_dn) == 18_800_640


def test_bf16_bytes_count_distinct_experts_once():
    wl = synth.WORKLOADS["flash_decode"]
    a = bench.algorithmic(wl, np.array([[1, 2, 3], [3, 2, 7]]), 2)
    b = bench.algorithmic(wl, np.array([[1, 2, 3], [3, 2, 8]]), 2)
    assert a["U"] == 4 and b["U"] == 4
    assert a["step_bytes"] == b["step_bytes"]
    per_expert = 3 * wl.H * wl.I * 2            # W1, W3, W2 in BF16
    c = bench.algorithmic(wl, np.array([[1, 2, 3], [4, 5, 6]]), 2)
    assert c["step_bytes"] - a["step_bytes"] == 2 * per_expert
    # flops: router plus 3 matrices per (token, expert) pair, shared expert included
    assert a["step_flops"] == 2 * 2 * wl.E * wl.H + (2 * 6 + wl.n_shared * 2) * 6 * wl.H * wl.I


def test_recorded_traffic_needs_matching_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "routed_expert_ffn_sqrtsoftplus_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.source_digest(["k.cu"])
    rec = {"w": {"kern": {"bytes_per_launch": 123, "sources": ["k.cu"], "sources_sha256_16": digest}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("w", "kern") == 123
    assert bench.recorded_traffic("w", "other") is None
    (csrc / "k.cu").write_text("kernel v2\n")
    assert bench.recorded_traffic("w", "kern") is None


def test_peaks_from_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks() == (6650.0, 1590.0, 1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        json.dumps({"hbm_gbs": 6472.5, "bf16_tflops": 1612.0, "bf16_tflops_sustained": 1401.0}))
    assert bench.peaks() == (6472.5, 1612.0, 1401.0, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6500, "bf16_tflops": 1600}))
    assert bench.peaks() == (6500.0, 1600.0, 1600.0, "measured")   # no sustained figure: the burst one


def test_roofline_fractions_use_the_measured_peaks(tmp_path, monkeypatch):
    """An HBM-bound kernel's frac is its algorithmic bytes per launch over its mean
    launch time, against the copy figure of MEASURED_PEAKS.json, and against the
    read-only probe when one was measured; a block-scaled contraction takes twice
    the measured BF16 rate."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}))
    hbm, tc, _, src = bench.peaks()
    prof = {"gemm_fused": (30.0, 20), "gemm_gateup_mx": (20.0, 10)}     # total ms, launches
    alg = {"kern": {"gemm_fused": (9.0e9, 1.0e12), "gemm_gateup_mx": (1.0e9, 6.0e12)},
           "step_bytes": 0.0, "step_flops": 0.0}
    r = bench.kernel_roofline("gemm_fused", prof, alg, hbm, tc, src, 7200.0, "nowhere")
    assert r["bound"] == "hbm" and r["peak"] == 6000.0 and r["peak_source"].startswith("measured")
    assert abs(r["achieved"] - 6000.0) < 1e-6 and abs(r["frac"] - 1.0) < 1e-9      # 9 GB in 1.5 ms
    assert abs(r["frac_of_read_peak"] - 6000.0 / 7200.0) < 1e-9 and r["traffic"] is None
    m = bench.kernel_roofline("gemm_gateup_mx", prof, alg, hbm, tc, src, 7200.0, "nowhere")
    assert m["bound"] == "tensor" and m["peak"] == 3000.0 and abs(m["achieved"] - 3000.0) < 1e-6   # 6 TFLOP in 2 ms
