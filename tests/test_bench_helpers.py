"""bench.py's host-side helpers, without a GPU: the clock-sample summary (throttle reasons and
the median SM clock that decide whether a run is kept), the DRAM-traffic lookup that only
trusts counters taken on the current kernel source, and the roofline peaks' fallback."""
import hashlib
import json
import os

import bench


def test_clock_summary_reports_median_max_and_reasons():
    c = bench.Clocks(0)
    c.out = "\n".join([
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1900, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ])
    s = c.summary()
    assert s == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c.out = "0, 1200, 1965, 500, 0x40, Active, Not Active, Active, Not Active"
    assert c.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples():
    c = bench.Clocks(0)
    c.out = ""
    assert c.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_traffic_only_for_the_source_it_was_measured_on(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"k": {"src": "kernel.cu", "src_sha": sha, "dram_bytes_per_launch": 12345}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("k") == 12345
    assert bench._traffic("other") is None
    src.write_text("// kernel v2\n")  # the kernel changed since the counters were taken
    assert bench._traffic("k") is None


def test_traffic_without_a_summary(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("k") is None


def test_peaks_measured_or_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._peaks() == (6650.0, 1590.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6529.4, "bf16_tflops": 1674.6}))
    assert bench._peaks() == (6529.4, 1674.6, "measured")


def test_committed_traffic_summary_names_existing_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        j = json.load(f)
    for key, e in j.items():
        assert os.path.exists(os.path.join(bench.ROOT, e["src"])), key
        assert e["dram_bytes_per_launch"] == sum(v["read"] + v["write"] for v in e["kernels"].values()), key
