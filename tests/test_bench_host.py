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


def test_recorded_traffic_is_tied_to_the_decode_sources(monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "decode_dram_traffic.json")))
    for key, ent in rec["configs"].items():
        h = ent["decode_source_hash"]
        monkeypatch.setattr(bench, "kernel_source_hash", lambda names=None: h)
        assert bench.recorded_traffic(key) == ent["bytes_per_launch"]
    assert bench.recorded_traffic("no such workload") is None
    # a capture taken on other sources is not reported
    monkeypatch.setattr(bench, "kernel_source_hash", lambda names=None: "0" * 16)
    for key in rec["configs"]:
        assert bench.recorded_traffic(key) is None


def test_kernel_source_hash_covers_every_source_file(tmp_path, monkeypatch):
    csrc = tmp_path / "paged_kv_cache_484_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("one")
    (csrc / "b.cuh").write_text("two")
    (tmp_path / "include").mkdir()
    (tmp_path / "include" / "pkv.h").write_text("api")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (csrc / "b.cuh").write_text("two ")
    assert bench.kernel_source_hash() != h0
    (csrc / "b.cuh").write_text("two")
    assert bench.kernel_source_hash() == h0
    # the decode hash covers only the named files and the public header
    d0 = bench.kernel_source_hash(("b.cuh",))
    (csrc / "a.cu").write_text("one ")
    assert bench.kernel_source_hash(("b.cuh",)) == d0
    (tmp_path / "include" / "pkv.h").write_text("api ")
    assert bench.kernel_source_hash(("b.cuh",)) != d0


def test_peak_falls_back_when_no_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6539.5}))
    assert bench.load_peak() == (6539.5, "measured")


def _timed_reuse_distance(nbytes, l2, K, warmup):
    """Replays the bench's warm-up and timed schedule as a list of the copies
    each step touches; returns, for every timed step, the bytes other steps
    moved since its copy was last touched (None: first touch)."""
    n, S = bench.copies_plan(nbytes, l2, K)
    warm_order, timed_order = bench.replay_order(K, S)
    uses = [k % n for k in range(max(warmup, n))]            # eager warm-up steps
    for length in warm_order:
        uses += [k % n for k in range(length)]
    t0 = len(uses)
    for length in timed_order:
        uses += [k % n for k in range(length)]
    assert len(uses) - t0 == K                                # exactly K timed steps
    last, dist = {}, []
    for i, c in enumerate(uses):
        if i >= t0:
            dist.append(None if c not in last else (i - last[c] - 1) * nbytes)
        last[c] = i
    return n, S, warm_order, timed_order, dist


def test_timed_steps_never_reread_what_l2_holds():
    """Every timed step reads a copy that at least 2 x L2 bytes of other steps
    have passed over since it was last used, for short and long timed regions
    (the driver's --steps 20 included) and small and large workloads."""
    l2 = 126 << 20
    for nbytes in (524_800, 4_202_496, 60 << 20, 283_000_000, 8_590_000_000):
        for K in (1, 3, 20, 50, 64, 65, 200, 2000):
            n, S, warm, timed, dist = _timed_reuse_distance(nbytes, l2, K, 5)
            if n == 1:
                assert nbytes >= 2 * l2
                continue
            assert all(d is not None and d >= 2 * l2 for d in dist), (nbytes, K, n, dist[:4])


def test_every_timed_graph_is_replayed_before_the_timed_region():
    for K in (1, 4, 16, 20, 33, 2000):
        for S in (1, 7, 16, 64, 83):
            warm, timed = bench.replay_order(K, S)
            assert sum(timed) == K
            assert set(timed) <= set(warm)
            assert warm[-1] == S          # the full graph runs last, over the highest copies
