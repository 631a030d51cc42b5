"""Host-side pieces of bench.py: the DRAM traffic figure is reported only while the decode
sources still match the ones the committed ncu capture was taken on."""
import os
import shutil

import pytest

import bench


def test_traffic_matches_the_committed_capture():
    n = 234_881_024
    t = bench.ncu_traffic_per_launch(n)
    if t is None:  # the kernel changed since the capture: the bench reports null, as it should
        pytest.skip("decode sources changed since the committed ncu capture")
    # DRAM bytes per weight read + written per launch: near the algorithmic ~3.34 (container
    # once, output once, part of it still in L2 at kernel end), not above it (no re-reads)
    assert 2.5 < t / n < 1.1 * 3.34
    assert abs(bench.ncu_traffic_per_launch(2 * n) - 2 * t) < 1.0


def test_traffic_is_null_once_a_decode_source_changes(tmp_path, monkeypatch):
    srcs = []
    for p in bench.DECODE_SOURCES:
        q = tmp_path / os.path.basename(p)
        shutil.copy(p, q)
        srcs.append(str(q))
    monkeypatch.setattr(bench, "DECODE_SOURCES", srcs)
    # a capture record keyed to these sources
    rec = tmp_path / "traffic.txt"
    rec.write_text(f"# test record\ndecode_source_sha256: {bench.decode_source_hash()}\n"
                   "dram_bytes_per_weight: 3.0\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.ncu_traffic_per_launch(1000) == 3000.0
    with open(srcs[0], "a") as fh:
        fh.write("\n")
    assert bench.ncu_traffic_per_launch(1000) is None


def test_traffic_is_null_without_the_file(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.txt"))
    assert bench.ncu_traffic_per_launch(1000) is None


def test_launch_times_by_tenth():
    # 50 steps: five at 135 us then five at 145 us per tenth -> the tenths show the step
    ms = [0.135] * 25 + [0.145] * 25
    assert bench.tenths(ms) == [135.0] * 5 + [145.0] * 5
    # fewer than ten steps: one entry per step
    assert bench.tenths([0.1354, 0.1361]) == [135.4, 136.1]


def test_clock_summary_reports_the_memory_side():
    c = bench.ClockSampler(0)
    c.samples, c.max_mhz = [1900, 1965, 1965], 1965
    c.reasons = {"sw_power_cap"}
    # side samples: memory clock, GPU temperature, HBM temperature (None: not reported), power
    c.side = [[3996, 40, None, 600.0], [3996, 44, None, 650.0], [3996, 46, None, 700.5]]
    s = c.summary()
    assert s["sm_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    assert s["mem_mhz"] == 3996
    assert s["gpu_temp_c"] == {"first": 40, "last": 46} and s["power_w"] == {"first": 600.0, "last": 700.5}
    assert "hbm_temp_c" not in s  # no answer from NVML: the key is left out, not faked
