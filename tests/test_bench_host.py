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


def test_traffic_written_from_ncu_csv_carries_the_device_code_hash(tmp_path, monkeypatch):
    csv = tmp_path / "fwd.csv"
    header = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream",'
              '"Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit",'
              '"Metric Value"\n')
    rows = []
    for i, (rd, wr) in enumerate(((400.0, 110.0), (402.0, 112.0))):
        for m, u, v in (("dram__bytes_read.sum", "Mbyte", rd), ("dram__bytes_write.sum", "Mbyte", wr),
                        ("gpu__time_duration.sum", "msecond", 3.1)):
            rows.append(f'"{i}","1","python","h","void sigattn::fwd_tiles_kernel<128, 0, 2, 3>(CUtensorMap_st)",'
                        f'"1","7","(640, 1, 1)","(64, 16, 2)","0","10.0","Command line profiler metrics",'
                        f'"{m}","{u}","{v}"\n')
    csv.write_text("==PROF== a line ncu prints before the table\n" + header + "".join(rows))
    out = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_PATH", str(out))
    d = bench.write_traffic([str(csv)], "cmd")
    assert d["fwd"] == 512_000_000 and d["_meta"]["launches"] == {"fwd": 2}
    assert d["_meta"]["source_sha256"] == bench.kernel_source_hash()
    assert bench._ncu_traffic("fwd") == 512_000_000
    assert bench._ncu_traffic("bwd_dkdv") is None
    # any edit of a device-code header invalidates the counters
    monkeypatch.setattr(bench, "DEVICE_SOURCES", bench.DEVICE_SOURCES[:-1])
    assert bench._ncu_traffic("fwd") is None


def test_device_code_hash_ignores_comments_but_not_code(tmp_path):
    """The traffic captures stay valid across comment edits of the device
    headers and are voided by any change of the code itself."""
    src = os.path.join(bench.ROOT, "padding_aware_sigmoid_b200", "csrc")
    base = bench.kernel_source_hash(src)
    for variant, same in (("comment", True), ("code", False)):
        d = tmp_path / variant
        d.mkdir()
        for name in bench.DEVICE_SOURCES:
            with open(os.path.join(src, name), encoding="utf-8") as f:
                text = f.read()
            if name == "sigmoid.cuh":
                text = ("// an added comment line\n/* and a block\n comment */" + text
                        if variant == "comment" else text.replace("0.5f", "0.25f", 1))
            (d / name).write_text(text, encoding="utf-8")
        assert (bench.kernel_source_hash(str(d)) == base) == same, variant


def test_gpus_2_starts_two_ranks_and_reports_them():
    """`bench.py --gpus 2` outside torchrun starts two ranks itself; on the
    reference arm rank 0 alone times the oracle and prints the line, and the
    line counts both ranks."""
    import subprocess
    import sys
    import oracle
    oracle.build()
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    ready = [ln for ln in r.stderr.splitlines() if ln.startswith("bench rank ")]
    assert sorted(ready) == ["bench rank 0 of 2 (local 0) ready", "bench rank 1 of 2 (local 1) ready"]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["impl"] == "reference" and d["value"] > 0
