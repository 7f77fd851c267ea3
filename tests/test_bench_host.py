"""Host-side pieces of bench.py, on CPU: the clock record's summary, the peaks
it divides by, and the gate that reports committed DRAM counters only while the
kernel sources match the ones they were taken on."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_clock_summary_takes_the_median_and_active_reasons():
    s = bench.ClockSampler(0)
    s.lines = [
        "1965, 1965, 812.1, Not Active, Not Active, Not Active, Active",
        "1800, 1965, 990.4, Not Active, Not Active, Not Active, Active",
        "1900, 1965, 950.0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    got = s.summary()
    assert got["sm_mhz"] == 1900.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"] and got["samples"] == 3
    s.lines = ["1965, 1965, 700, Active, Not Active, Active, Not Active"]
    assert s.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    s.lines = []
    assert s.summary()["reasons"] == ["unsampled"]


def test_peaks_come_from_the_measured_file():
    pk = bench.peaks()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        assert pk["source"] == "fallback" and pk["bf16"] == 1590.0
        return
    d = json.load(open(path))
    assert pk["source"] == "measured"
    assert pk["bf16"] == float(d["bf16_tflops"]) and pk["hbm"] == float(d["hbm_gbs"])


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(monkeypatch):
    h = bench.kernel_source_hash()
    assert h == bench.kernel_source_hash() and len(h) == 64
    stored = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    if stored["_meta"]["source_sha256"] == h:
        for k in ("fwd", "bwd_dq", "bwd_dkdv"):
            assert bench._ncu_traffic(k) == stored[k]
            # the counters never exceed the kernel's compulsory bytes by much
            assert stored[k] <= 1.05 * stored["_meta"]["algorithmic_bytes"][k]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 64)
    assert bench._ncu_traffic("bwd_dkdv") is None
