"""Host-side helpers of bench.py (CPU): the ncu DRAM traffic a bench line
reports is taken only when the committed capture was made on the current
kernel sources, and the peak falls back to the stated figure when no
measured peaks file exists."""
from __future__ import annotations

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_recorded_traffic_is_tied_to_the_kernel_sources(monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "decode_dram_traffic.json")))
    h = rec["kernel_source_hash"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: h)
    for key, ent in rec["configs"].items():
        assert bench.recorded_traffic(key) == ent["bytes_per_launch"]
    assert bench.recorded_traffic("no such workload") is None
    # a capture taken on other sources is not reported
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    for key in rec["configs"]:
        assert bench.recorded_traffic(key) is None


def test_kernel_source_hash_covers_every_source_file(tmp_path, monkeypatch):
    csrc = tmp_path / "paged_kv_cache_484_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("one")
    (csrc / "b.cuh").write_text("two")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (csrc / "b.cuh").write_text("two ")
    assert bench.kernel_source_hash() != h0
    (csrc / "b.cuh").write_text("two")
    assert bench.kernel_source_hash() == h0


def test_peak_falls_back_when_no_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6539.5}))
    assert bench.load_peak() == (6539.5, "measured")
