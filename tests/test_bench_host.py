"""Host-side pieces of bench.py that decide what a measurement line says:
the clock summary (which decides whether a run is rejected), the peaks it
divides by, and the scan-traffic lookup's source check.  CPU only."""
import json
import os

import bench


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.lines = list(lines)
    return s


def test_clock_summary_median_max_and_reasons():
    lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1890, 1965, 990.3, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = _sampler(lines).summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_reports_every_slowdown_reason():
    line = "0, 1500, 1965, 400.0, 0x68, Active, Active, Active, Not Active"
    s = _sampler([line]).summary()
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples():
    s = _sampler([]).summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and s["reasons"] == ["unsampled"]


def test_peaks_fall_back_when_the_measured_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    p, src = bench.load_peaks()
    assert src == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"hbm_gbs": 6541.8, "bf16_tflops": 1624.0}))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    p, src = bench.load_peaks()
    assert src == "measured" and p["hbm_gbs"] == 6541.8


def test_scan_traffic_only_for_the_sources_it_was_measured_on(tmp_path, monkeypatch):
    # a copy of the scan sources and a traffic file keyed to their hash
    for rel in bench.SCAN_SOURCES:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(bench.ROOT, rel), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash(bench.SCAN_SOURCES)
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(
        json.dumps({"w": {"scan": {"dram_bytes_per_launch": 123, "source_hash": h}}}))
    assert bench.scan_traffic("w") == 123
    assert bench.scan_traffic("other") is None
    # any change to a scan source withdraws the figure
    src = tmp_path / bench.SCAN_SOURCES[0]
    src.write_bytes(src.read_bytes() + b"\n// changed\n")
    assert bench.scan_traffic("w") is None


def test_rank_seeds_differ_per_rank_and_repeat():
    from sparse_attention_decode_scan_b200 import synth
    spec = synth.WORKLOADS[synth.DECODE_B32]
    seeds = [bench.rank_seed(spec, r) for r in range(8)]
    assert len(set(seeds)) == 8
    assert seeds == [bench.rank_seed(spec, r) for r in range(8)]
