"""Host-side logic of bench.py with two ranks on the CPU (gloo): the step time
is the maximum over ranks, the whole-job value counts every rank's work
(weak scaling: each rank runs its own copy of the workload, no collective on
the data path), and only rank 0 prints.  The reference arm under the
launcher runs on rank 0 alone; the other rank exits 0 without work."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench

    dist = bench.init_dist(world, rank, backend="gloo")
    # per-rank step times: the job is as slow as its slowest rank
    t = [1.5, 2.5][rank]
    tmax = bench.max_over_ranks(t, world, torch.device("cpu"))
    bench.barrier(world, torch.device("cpu"))
    results[rank] = tmax
    dist.destroy_process_group()


def test_step_time_is_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert results[0] == results[1] == 2.5


def test_reference_arm_under_launcher_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--cpu-seconds", "1", "--config", "1"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_algorithmic_bytes_of_the_named_steps():
    """The bench's byte count is every decoded token's K and V row once per KV
    head plus q in and out: 2049 tokens x 8 heads x 64 x 2 (K, V) x 2 bytes +
    32 heads x 64 x (2 + 2) bytes for the batch-1 Llama step."""
    sys.path.insert(0, ROOT)
    import torch
    import bench
    from paged_kv_cache_484_b200 import workloads as W
    assert bench.step_bytes(W.make_config(2), torch.bfloat16) == 2049 * 8 * 64 * 2 * 2 + 32 * 64 * 4
    assert bench.step_bytes(W.make_config(1), torch.float32) == 257 * 4 * 64 * 2 * 4 + 4 * 64 * 8
