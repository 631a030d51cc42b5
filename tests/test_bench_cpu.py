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
