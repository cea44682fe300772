"""CPU tests of bench.py's host logic: the clock-record summary that decides whether a run is
throttled, the GPU index mapping, the peaks and the source-hash gate on committed traffic."""
import json
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_clock_summary_median_max_and_reasons():
    lines = ["1965, 1965, Not Active, Not Active, Not Active, Not Active",
             "1800, 1965, Not Active, Not Active, Not Active, Active",
             "1950, 1965, Not Active, Not Active, Not Active, Not Active",
             "[N/A], 1965, Not Active, Not Active, Not Active, Not Active",   # not a number: skipped
             "1965, 1965, Active"]                                            # wrong field count: skipped
    got = bench.ClockSampler.summarize(lines)
    assert got == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_summary_reports_thermal_and_hw_slowdown():
    got = bench.ClockSampler.summarize(["1200, 1965, Active, Not Active, Active, Not Active"])
    assert got["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.ClockSampler.summarize([]) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_physical_gpu_follows_visible_devices(monkeypatch):
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3, 5")
    assert bench.physical_gpu(0) == "3" and bench.physical_gpu(1) == "5"
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench.physical_gpu(2) == "2"


def test_peaks_come_from_the_measured_file():
    p = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        assert bench.peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
        return
    with open(p) as f:
        d = json.load(f)
    assert bench.peaks() == (float(d["hbm_gbs"]), "measured")
    if "bf16_tflops" in d:
        assert bench.tensor_peak() == float(d["bf16_tflops"])


def test_committed_traffic_is_gated_by_the_kernel_source_hash(monkeypatch):
    import json
    prof = os.path.join(bench.ROOT, "profiles", "k_qgemv_tinyllama_decode.json")
    rec = json.load(open(prof))
    want = int(rec["traffic_bytes_per_launch"])
    if rec["kernel_source_hash"] == bench.kernel_source_hash():
        assert bench.committed_traffic() == want
    else:
        assert bench.committed_traffic() is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.committed_traffic() is None  # another kernel source: no traffic figure
