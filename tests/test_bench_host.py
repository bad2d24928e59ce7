"""Host logic of bench.py, no GPU: the clock summary keeps the samples of the
timed region, the recorded DRAM traffic is reported only for the kernel source
it was captured on, and every bench kernel has a record."""
import json
import os

import bench


def test_clock_summary_uses_the_timed_region():
    c = bench.ClockSampler(0)
    c.samples = [(0.0, 1965.0, 1965.0, []), (1.0, 1800.0, 1965.0, ["sw_power_cap"]),
                 (1.5, 1850.0, 1965.0, ["sw_power_cap"]), (2.0, 1900.0, 1965.0, []), (9.0, 1200.0, 1965.0, ["hw_slowdown"])]
    c.mark(0.9, 2.1)
    s = c.summary()
    assert s["window"] == "timed region" and s["samples"] == 3
    assert s["sm_mhz"] == 1850.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]  # the hw_slowdown sample lies outside the timed region


def test_clock_summary_without_samples_in_the_region_falls_back_to_the_run():
    c = bench.ClockSampler(0)
    c.samples = [(0.0, 1965.0, 1965.0, [])]
    c.mark(5.0, 6.0)
    s = c.summary()
    assert s["window"].startswith("benchmark run") and s["samples"] == 1
    assert bench.ClockSampler(0).summary() is None


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    key = "wkv4_bwd_kernel"
    good = bench._kernel_source_hash(key)
    assert good == bench._kernel_source_hash(key)  # stable
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps({key: {"dram_bytes_per_launch": 123, "source_hash": good}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the hash reads the sources under ROOT: point it back at the repository's sources
    monkeypatch.setattr(bench, "_kernel_source_hash", lambda k: good)
    assert bench._recorded_traffic(key) == 123
    monkeypatch.setattr(bench, "_kernel_source_hash", lambda k: "0" * 16)
    assert bench._recorded_traffic(key) is None


def test_every_bench_kernel_has_a_traffic_record():
    # a record whose source hash no longer matches is reported as null by the bench (above)
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for key in bench._TRAFFIC_SOURCES:
        assert key in rec, key
        assert len(rec[key]["source_hash"]) == 16
        assert rec[key]["dram_bytes_per_launch"] > 0
        assert "--clock-control none" in rec[key]["command"]
