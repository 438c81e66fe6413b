#!/usr/bin/env python3
"""Benchmark of the paged decode step: kv_append + paged_attention_decode.

Default run: one JSON line for the long-context workload (16 sequences x
131072 cached tokens + 1 appended, 32 query / 8 KV heads, head_dim 128,
block size 16, bf16, 1 % of key rows x8, split-K with a partition combine:
8.6 GB of K/V per step), the largest single-GPU workload and the cleanest
HBM roofline case.  The same line carries, under ``per_config``, the other
bf16 workloads timed the same way (same K and W): the batch-1 Llama-3.2-1B
layer step, the ragged batch of 64 and the 256-sequence prefix-sharing mix.
``--config N`` times workload N alone.  Metric: achieved HBM GB/s of the
step's algorithmic bytes (K/V of every context token + q + out), with
seq-steps/s alongside.

Timing: W warm-up steps, then exactly K timed steps back to back between one
pair of CUDA events on the launch stream (synchronised on both sides).  The
steps are replays of CUDA graphs that captured the library call(s) of
consecutive steps, so host-side marshalling does not set the pace; every
graph the timed region replays has been replayed before it.  The inputs are
larger than L2: when one copy of the workload touches less than twice the L2
size per step, the bench holds enough device-side copies (like the per-layer
caches of a model) that every timed step reads a copy no step of the last
2 x L2 bytes touched.  ``isolated_step`` is the older, pessimistic figure:
one step at a time, L2 flushed before it, each step between its own pair of
events (whose own cost, a few microseconds, it includes).  Under torchrun
every rank runs its own copy of the workload (weak scaling, no collective on
the data path); the step time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only); it is the deliberately slow definition
the CUDA path is checked against, not an optimised baseline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode-attention achieved HBM GB/s (% of B200 peak); seq-steps/sec"
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 512 << 20
HEADLINE_CONFIG = 5
SECONDARY_CONFIGS = (2, 3, 4)
# the oracle's bounded sample: whole sequences while their K/V stay within this
SAMPLE_KV_BYTES = 1_100_000_000


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=None, choices=[1, 2, 3, 4, 5],
                    help="time this workload alone (default: the long-context workload, "
                         "with the other bf16 workloads under per_config)")
    ap.add_argument("--no-secondary", action="store_true",
                    help="default run: leave out the per_config workloads")
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="keep only the first N sequences of the workload (small profiler "
                         "captures of the same kernel)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--out-dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--partition-tokens", type=int, default=0)
    ap.add_argument("--copies", type=int, default=0,
                    help="device-side copies of the workload (0: enough to exceed L2)")
    ap.add_argument("--simt", action="store_true", help="bf16: CUDA-core decode kernel")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding window: each query attends to the last W tokens")
    ap.add_argument("--kv-dtype", default="native", choices=["native", "e4m3"],
                    help="e4m3: the workload's cache as an 8-bit cache (per-tensor scales), "
                         "stepped by decode_step_e4m3 (kv_append_e4m3 + "
                         "paged_attention_decode_e4m3 with --two-calls)")
    ap.add_argument("--two-calls", action="store_true",
                    help="time kv_append + paged_attention_decode as two launches instead of "
                         "the single-launch decode_step")
    ap.add_argument("--cascade", action="store_true",
                    help="two calls, the decode as paged_attention_decode_cascade over the "
                         "workload's prefix groups (config 4)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--prefill", type=int, default=0, metavar="C",
                    help="time chunked prefill instead: the last C context tokens of every "
                         "sequence of the workload attend causally to its paged cache")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local, backend="nccl"):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        kw = dict(backend=backend, timeout=datetime.timedelta(seconds=120))
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(**kw)
    return dist


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def esize(dt):
    return 2 if dt == torch.bfloat16 else 4


def step_bytes(w, out_dtype, window=0) -> int:
    """Algorithmic bytes of one decode call: every attended context token's K
    and V row once per KV head (at the cache's element size), plus q read and
    out written.  With a sliding window only the last ``window`` tokens of a
    context count."""
    lens = w.decode_lens.to(torch.int64)
    if window:
        lens = lens.clamp(max=window)
    L = int(lens.sum().item())
    kv = L * w.Hkv * w.d * 2 * w.k_cache.element_size()
    qo = w.B * w.Hq * w.d * (esize(w.dtype) + esize(out_dtype))
    return kv + qo


def load_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The sources a decode call's kernels and their launch plan are built from
# (the chunked prefill and the cascade's shared-prefix pass live elsewhere).
DECODE_SOURCES = ("paged_decode.cu", "pkv_api.cu", "pkv_device.cuh", "pkv_internal.h")


def kernel_source_hash(names=None) -> str:
    """Hash of the library's CUDA sources (``names``: only those files of
    csrc/, plus the public header; default: every file)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_484_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if names is not None and name not in names:
            continue
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    if names is not None:
        with open(os.path.join(ROOT, "include", "pkv.h"), "rb") as f:
            h.update(b"pkv.h" + f.read())
    return h.hexdigest()[:16]


def software_versions() -> dict:
    """Versions the numbers were taken with (NVML read only)."""
    v = {"torch": torch.__version__, "cuda_runtime": torch.version.cuda,
         "kernel_sources": kernel_source_hash(),
         "decode_sources": kernel_source_hash(DECODE_SOURCES)}
    try:
        # the git commit, where the checkout carries its history
        r = subprocess.run(["git", "-C", ROOT, "rev-parse", "--short", "HEAD"],
                           capture_output=True, text=True, timeout=10)
        if r.returncode == 0 and r.stdout.strip():
            v["commit"] = r.stdout.strip()
    except Exception:
        pass
    try:
        import pynvml
        pynvml.nvmlInit()
        d = pynvml.nvmlSystemGetDriverVersion()
        v["driver"] = d.decode() if isinstance(d, bytes) else d
    except Exception:
        pass
    return v


def recorded_traffic(cfg):
    """DRAM bytes per decode launch from the committed ncu capture, if it was
    taken on the current decode sources (else None).  ``cfg``: the config
    number, or e.g. "3_e4m3" for its 8-bit cache.  A workload captured on a
    smaller batch of the same kernel is recorded already scaled to the full
    launch."""
    path = os.path.join(ROOT, "profiles", "decode_dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    ent = rec.get("configs", {}).get(str(cfg))
    if ent is None or ent.get("decode_source_hash") != kernel_source_hash(DECODE_SOURCES):
        return None
    return ent.get("bytes_per_launch")


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML (read only) while the
    timed region runs.  The first sample is taken before ``__enter__``
    returns, so even a region shorter than the polling period has one."""

    REASONS = {
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._first = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False

    def _sample(self):
        nv = self._nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for bit, name in self.REASONS.items():
                if mask & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        self._sample()
        self._first.set()
        while not self._stop.wait(self._period):
            self._sample()
        self._sample()

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
            self._first.wait(5.0)
        return self

    def __exit__(self, *exc):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def config_block(cfg, w, out_dtype, P, NP, simt, two_calls=False):
    from paged_kv_cache_484_b200 import workloads as W
    s = W.config_summary(cfg)
    name = w.name if w.name.startswith(W.CONFIG_NAMES[cfg]) else W.CONFIG_NAMES[cfg]
    if w.k_cache.dtype == torch.uint8:
        return {
            "workload": name + "_e4m3cache",
            "batch_seqs": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d,
            "context": s["ctx"], "tokens_decoded": int(w.decode_lens.to(torch.int64).sum().item()),
            "block_size": w.block_size, "pool_blocks": w.num_blocks,
            "kv_dtype": "e4m3 (per-tensor scales: max|x| / 448)",
            "kv_scales": list(w.meta.get("e4m3_scales", ())),
            "out_dtype": "bf16" if out_dtype == torch.bfloat16 else "f32",
            "partition_tokens": P, "max_partitions": NP, "decode_kernel": "mma_f16 (e4m3 pages)",
            "step": "two calls (kv_append_e4m3, paged_attention_decode_e4m3)" if two_calls
                    else "one launch (decode_step_e4m3: append fused into the decode kernel)",
        }
    return {
        "workload": name,
        "batch_seqs": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d,
        "context": s["ctx"], "tokens_decoded": int(w.decode_lens.to(torch.int64).sum().item()),
        "block_size": w.block_size, "pool_blocks": w.num_blocks,
        "kv_dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "out_dtype": "bf16" if out_dtype == torch.bfloat16 else "f32",
        "partition_tokens": P, "max_partitions": NP,
        "decode_kernel": "simt" if (simt or w.dtype == torch.float32) else "mma_bf16",
        "step": "two calls (kv_append, paged_attention_decode)" if two_calls
                else "one launch (decode_step: append fused into the decode kernel)",
    }


# ---------------------------------------------------------------- timing plan

def copies_plan(nbytes: int, l2_bytes: int, K: int, forced: int = 0):
    """How many device-side copies of the workload the bench holds, and how
    many consecutive steps one CUDA graph captures (S).

    A step whose inputs exceed twice the L2 size runs on one copy.  Otherwise
    ``n_min`` copies put 2 x L2 bytes of other steps between two uses of the
    same copy.  Graphs: one of S steps over copies 0..S-1 and, when S does not
    divide K, one of the K mod S first steps; the timed region replays the
    first K // S times, then the second.  When K is small, K extra copies
    keep even the tail graph's copies out of L2: the warm-up replays of both
    graphs end with ``n - K >= n_min`` steps on other copies."""
    if forced:
        n = forced
        return n, (n if n > 1 else min(K, 16))
    n_min = 1 if nbytes >= 2 * l2_bytes else 1 + math.ceil(2 * l2_bytes / nbytes)
    if n_min == 1:
        return 1, min(K, 16)
    n = n_min + K if K <= 4 * n_min else n_min
    return n, n


def replay_order(K: int, S: int):
    """Graph replays: (warm-up, timed), as lists of graph lengths in steps.
    The warm-up replays the tail graph (if any) and then the full graph, so
    every graph the timed region replays has run once (its first launch pays
    the graph's upload) and the last warm-up steps use the highest copies."""
    tail = K % S
    warm = ([tail] if tail else []) + [S]
    timed = [S] * (K // S) + ([tail] if tail else [])
    return warm, timed


# ---------------------------------------------------------------- oracle arm

def oracle_sample(w, window: int = 0):
    """The oracle's bounded sample of a workload: whole sequences, in order,
    while their K/V stay within SAMPLE_KV_BYTES (at least one).  Returns the
    sequence indices and the fraction of the step's attended tokens they
    hold."""
    lens = w.decode_lens.cpu().tolist()
    row = w.Hkv * w.d * 2 * w.k_cache.element_size()
    seqs, kv = [], 0
    for b in range(w.B):
        if seqs and kv + lens[b] * row > SAMPLE_KV_BYTES:
            break
        seqs.append(b)
        kv += lens[b] * row
    att = [min(L, window) if window else L for L in lens]
    return seqs, sum(att[b] for b in seqs) / max(1, sum(att))


def oracle_step(sub, nthreads: int, e4m3_scales=None, window: int = 0):
    """One oracle append + decode over the sample; returns its seconds.  The
    append writes the same rows every time, so only q (rotated in place) is
    restored between repetitions."""
    import oracle
    q = sub.q.clone()
    t0 = time.perf_counter()
    if e4m3_scales is not None:
        ks, vs = e4m3_scales
        oracle.kv_append_e4m3(q, sub.k_new, sub.v_new, sub.positions, sub.slots, sub.k_cache,
                              sub.v_cache, sub.theta, ks, vs)
        oracle.paged_attention_decode_e4m3(q, sub.k_cache, sub.v_cache, sub.tables,
                                           sub.decode_lens, sub.scale, ks, vs, nthreads=nthreads,
                                           window=window)
    else:
        oracle.kv_append(q, sub.k_new, sub.v_new, sub.positions, sub.slots, sub.k_cache,
                         sub.v_cache, sub.theta)
        oracle.paged_attention_decode(q, sub.k_cache, sub.v_cache, sub.tables, sub.decode_lens,
                                      sub.scale, nthreads=nthreads, window=window)
    return time.perf_counter() - t0


def time_oracle(sub, seconds: float, nthreads: int, e4m3_scales=None, window: int = 0):
    """Oracle steps over the sample, repeated until ~``seconds`` of CPU time."""
    reps, t_total = 0, 0.0
    while t_total < seconds or reps == 0:
        t_total += oracle_step(sub, nthreads, e4m3_scales, window)
        reps += 1
    return t_total / reps, reps


def run_reference(args):
    """The fp64 oracle, as it stands, on the host cores: W untimed and K timed
    steps, each one append + decode pass over the bounded sample of the same
    seeded workload (generated on the GPU when there is one, as the CUDA arm
    generates it; no library kernel runs)."""
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    from paged_kv_cache_484_b200 import workloads as W
    cfg = args.config or HEADLINE_CONFIG
    out_dtype = torch.bfloat16 if args.out_dtype == "bf16" else torch.float32
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    w = W.make_config(cfg, device=dev, num_seqs=args.num_seqs)
    seqs, frac = oracle_sample(w)
    sub = W.extract_sequences(w, seqs)
    nbytes = step_bytes(w, out_dtype)
    del w
    if dev.type == "cuda":
        torch.cuda.empty_cache()
    nthreads = os.cpu_count() or 1
    for _ in range(max(0, args.warmup)):
        oracle_step(sub, nthreads)
    K = max(1, args.steps)
    per_step = sum(oracle_step(sub, nthreads) for _ in range(K)) / K
    value = nbytes * frac / per_step / 1e9
    B = W.config_summary(cfg)["B"] if args.num_seqs is None else args.num_seqs
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": K, "warmup": max(0, args.warmup),
        "ms_per_step": round(per_step * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "seq_steps_per_s": round(len(seqs) / per_step, 3),
        "config": {"workload": W.CONFIG_NAMES[cfg], **W.config_summary(cfg),
                   **({"num_seqs": args.num_seqs} if args.num_seqs is not None else {})},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": nthreads,
                         "kind": "oracle",
                         "sample": f"sequences {seqs[0]}..{seqs[-1]} ({len(seqs)} of {B}, "
                                   f"{100 * frac:.1f} % of the step's K/V), one fp64 append + "
                                   f"decode pass over them per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- CUDA arm

def measure(cfg, args, device, world, local, rank, full: bool):
    """Time workload ``cfg`` as the bench's step.  Returns the JSON fields of
    its line (``full``: with the end-to-end figure and the CPU baseline)."""
    import paged_kv_cache_484_b200 as pkv
    from paged_kv_cache_484_b200 import workloads as W

    out_dtype = torch.bfloat16 if args.out_dtype == "bf16" else torch.float32
    w = W.make_config(cfg, device=device, num_seqs=args.num_seqs)
    e4m3 = args.kv_dtype == "e4m3"
    two_calls = args.two_calls
    ks8 = vs8 = None
    if e4m3:
        if w.dtype != torch.bfloat16:
            raise SystemExit("--kv-dtype e4m3 takes a bf16 workload (configs 2-5)")
        k8, v8, ks8, vs8 = W.e4m3_cache(w)
        # the library's 8-bit cache: one [K | V] region per page, one buffer
        w.k_cache = W.e4m3_pack(k8, v8)
        w.v_cache = w.k_cache
        del k8, v8
        w.meta["e4m3_scales"] = (ks8, vs8)
        torch.cuda.empty_cache()
    kv_dt = torch.uint8 if e4m3 else w.dtype
    host_inputs = None
    if full and not args.no_e2e:
        # pristine copies of the per-step inputs, in pinned host memory
        host_inputs = {k: v.cpu().pin_memory() for k, v in dict(
            q=w.q, k_new=w.k_new, v_new=w.v_new, positions=w.positions,
            slot_mapping=w.slot_mapping, block_tables=w.block_tables,
            decode_lens=w.decode_lens).items()}
    sample = None
    if full and rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle's bounded sample, copied to the host before any step
        seqs, frac = oracle_sample(w, args.window)
        sample = (W.extract_sequences(w, seqs), frac)

    P = args.partition_tokens or pkv.decode_partition_tokens(w.B, w.Hq, w.Hkv, w.d, w.max_blocks,
                                                              kv_dtype=kv_dt)
    NP = math.ceil(w.max_blocks * w.block_size / P)
    ws_bytes = pkv.decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks, kv_dtype=kv_dt,
                                         partition_tokens=P)
    # the calls get the caller's choice: 0 lets the library pick, which under
    # a sliding window can be shorter than the planned P (the same workspace)
    P_call = args.partition_tokens
    ws = pkv.new_workspace(ws_bytes, device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    nbytes = step_bytes(w, out_dtype, args.window)

    K = args.steps
    Wu = max(3, args.warmup)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    ncopies, S = copies_plan(nbytes, l2, K, args.copies)
    # Per-layer tensors (q, the new rows, the caches) get their own copy; the
    # step's metadata (positions, slots, block tables, context lengths) is one
    # set shared by all copies, as one decode step's metadata is shared by all
    # layers of a model.
    layer_fields = ("q", "k_new", "v_new", "k_cache") + (() if e4m3 else ("v_cache",))
    step_fields = ("positions", "slot_mapping", "block_tables", "decode_lens")
    copies = [dict((f, getattr(w, f)) for f in layer_fields + step_fields)]
    for _ in range(ncopies - 1):
        copies.append(dict([(f, getattr(w, f).clone()) for f in layer_fields] +
                           [(f, getattr(w, f)) for f in step_fields]))
    if e4m3:
        for c in copies:
            c["v_cache"] = c["k_cache"]  # the packed 8-bit cache holds both
    outs = [torch.empty((w.B, w.Hq, w.d), dtype=out_dtype, device=device) for _ in range(ncopies)]

    cascade = args.cascade
    if cascade:
        if e4m3:
            raise SystemExit("--cascade takes the bf16 cache")
        if w.meta.get("prefix_group", 0) <= 1:
            raise SystemExit("--cascade needs a workload with prefix groups (config 4)")
        two_calls = True
        grp = int(w.meta["prefix_group"])
        group_start = torch.tensor(list(range(0, w.B, grp)) + [w.B], dtype=torch.int32,
                                   device=device)
        cached = w.cached_lens.to(torch.int64)
        shared_tokens = (torch.minimum(cached // 16,
                                       torch.full_like(cached, w.meta["prefix_tokens"] // 16))
                         * 16).to(torch.int32)
        ws = pkv.new_workspace(pkv.decode_cascade_workspace_size(
            w.B, w.Hq, w.Hkv, w.d, w.max_blocks, partition_tokens=P), device)
    fused = not two_calls
    # decode kernel, plus the partition combine unless the split contexts
    # are merged inside thread-block clusters (the library decides)
    kernels_per_decode = pkv.decode_launches(w.B, w.Hq, w.Hkv, w.d, w.max_blocks, kv_dtype=kv_dt,
                                             out_dtype=out_dtype, partition_tokens=P,
                                             force_simt=args.simt, fused=fused)
    if kernels_per_decode not in (1, 2):
        raise SystemExit("decode_launches: no answer from the library")
    if cascade:
        kernels_per_decode = 3     # decode, shared-prefix pass, combine
    launches_per_step = kernels_per_decode + (0 if fused else 1)

    def append(c):
        if fused:
            return
        if e4m3:
            pkv.kv_append_e4m3(c["q"], c["k_new"], c["v_new"], c["positions"], c["slot_mapping"],
                               c["k_cache"], w.rope_theta, ks8, vs8, device_error=err)
        else:
            pkv.kv_append(c["q"], c["k_new"], c["v_new"], c["positions"], c["slot_mapping"],
                          c["k_cache"], c["v_cache"], w.rope_theta, device_error=err)

    def decode(c, out):
        if e4m3 and fused:
            pkv.decode_step_e4m3(c["q"], c["k_new"], c["v_new"], c["positions"],
                                 c["slot_mapping"], c["k_cache"], c["block_tables"],
                                 c["decode_lens"], w.rope_theta, w.scale, ks8, vs8, out,
                                 workspace=ws, partition_tokens=P_call, device_error=err,
                                 sliding_window=args.window)
        elif e4m3:
            pkv.paged_attention_decode_e4m3(c["q"], c["k_cache"], c["block_tables"],
                                            c["decode_lens"], w.scale, ks8, vs8, out,
                                            workspace=ws, partition_tokens=P_call, device_error=err,
                                            sliding_window=args.window)
        elif fused:
            pkv.decode_step(c["q"], c["k_new"], c["v_new"], c["positions"], c["slot_mapping"],
                            c["k_cache"], c["v_cache"], c["block_tables"], c["decode_lens"],
                            w.rope_theta, w.scale, out, workspace=ws, partition_tokens=P_call,
                            force_simt=args.simt, device_error=err, sliding_window=args.window)
        elif cascade:
            pkv.paged_attention_decode_cascade(c["q"], c["k_cache"], c["v_cache"],
                                               c["block_tables"], c["decode_lens"], group_start,
                                               shared_tokens, grp, w.scale, out, workspace=ws,
                                               partition_tokens=P_call, force_simt=args.simt,
                                               device_error=err, sliding_window=args.window)
        else:
            pkv.paged_attention_decode(c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                                       c["decode_lens"], w.scale, out, workspace=ws,
                                       partition_tokens=P_call, force_simt=args.simt,
                                       device_error=err, sliding_window=args.window)

    def step(k):
        c = copies[k % ncopies]
        append(c)
        decode(c, outs[k % ncopies])

    stream = torch.cuda.current_stream(device)
    for k in range(max(Wu, ncopies)):
        step(k)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"device error flag {int(err.item()):#x} during warm-up")

    def timed(K_, body):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier(world, device)
        torch.cuda.synchronize()
        e0.record(stream)
        for k in range(K_):
            body(k)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world, device)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K_

    # The timed steps are replays of CUDA graphs that captured S consecutive
    # steps (one per copy when there are copies), launches and programmatic
    # dependencies as the library issues them: the host's per-call
    # marshalling (tens of microseconds in Python) then does not set the pace
    # of a step whose kernels take a few microseconds, and the next step's
    # decode launches while the current one ends, as consecutive layers
    # would.  K = q S + r steps are q replays of the S-step graph and one of
    # an r-step graph; both are replayed once before the timed region.
    warm_order, timed_order = replay_order(K, S)

    def capture(body, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for k in range(n):
                body(k)
        return g

    def graphs_for(body):
        gs = {n: capture(body, n) for n in set(warm_order + timed_order)}
        torch.cuda.synchronize()
        return gs

    def warm(gs):
        for n in warm_order:
            gs[n].replay()
        torch.cuda.synchronize()

    def replay(gs):
        def run(_):
            for n in timed_order:
                gs[n].replay()
        return run

    step_g = graphs_for(step)
    decode_g = step_g if fused else graphs_for(lambda k: decode(copies[k % ncopies],
                                                                outs[k % ncopies]))

    # kv_append alone (not part of the roofline claim): the same graph scheme
    def append_only(k):
        c = copies[k % ncopies]
        if e4m3:
            pkv.kv_append_e4m3(c["q"], c["k_new"], c["v_new"], c["positions"], c["slot_mapping"],
                               c["k_cache"], w.rope_theta, ks8, vs8, device_error=err)
        else:
            pkv.kv_append(c["q"], c["k_new"], c["v_new"], c["positions"], c["slot_mapping"],
                          c["k_cache"], c["v_cache"], w.rope_theta, device_error=err)

    append_g = graphs_for(append_only)

    warm(step_g)
    with ClockSampler(local) as clocks:
        step_ms = timed(1, replay(step_g)) / K
    decode_ms = step_ms
    if not fused:
        # the decode call alone (the same call as the step when it is fused)
        warm(decode_g)
        decode_ms = timed(1, replay(decode_g)) / K
    warm(append_g)
    append_ms = max_over_ranks(timed(1, replay(append_g)) / K, world, device)
    step_ms_max = max_over_ranks(step_ms, world, device)
    decode_ms_max = max_over_ranks(decode_ms, world, device)
    if int(err.item()) != 0:
        raise SystemExit(f"device error flag {int(err.item()):#x} during timing")
    del step_g, decode_g, append_g

    value = world * nbytes / (step_ms_max * 1e-3) / 1e9
    peak, peak_src = load_peak()
    achieved = nbytes / (decode_ms_max * 1e-3) / 1e9

    # isolated steps: L2 flushed before each, each between its own events
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush_r = torch.ones(FLUSH_BYTES // 2, dtype=torch.uint8, device=device)

    def flush_l2():
        flush_w.zero_()      # evict: write more than L2 holds
        flush_r.max()        # then read more than L2 holds, so no dirty line is left

    Ki = max(1, min(K, 200))
    evi = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ki)]
    for k in range(Ki):
        flush_l2()
        evi[k][0].record(stream)
        step(0)
        evi[k][1].record(stream)
    torch.cuda.synchronize()
    iso_each = sorted(a.elapsed_time(b) for a, b in evi)
    iso_ms = max_over_ranks(sum(iso_each) / Ki, world, device)
    del flush_w, flush_r

    # end to end: pinned host inputs -> device, the call(s), out -> pinned host,
    # back to back over the same copies
    e2e = None
    if host_inputs is not None:
        out_host = torch.empty(outs[0].shape, dtype=out_dtype, pin_memory=True)
        # the step's inputs packed into one pinned host buffer (16-byte aligned
        # fields) and copied into one device buffer whose views the call reads:
        # one H2D copy per step instead of seven
        offs, size = {}, 0
        for name, t in host_inputs.items():
            offs[name] = size
            size += (t.numel() * t.element_size() + 15) // 16 * 16

        def view(buf, name):
            t = host_inputs[name]
            nb = t.numel() * t.element_size()
            return buf[offs[name]:offs[name] + nb].view(t.dtype).view(t.shape)

        hbuf = torch.zeros(size, dtype=torch.uint8, pin_memory=True)
        dbuf = torch.empty(size, dtype=torch.uint8, device=device)
        for name, t in host_inputs.items():
            view(hbuf, name).copy_(t)
        dev_in = {name: view(dbuf, name) for name in host_inputs}
        h2d = size
        d2h = out_host.numel() * out_host.element_size()

        if fused and not e4m3 and not args.window:
            # the fused step prepared once per layer copy (as a model's layer
            # loop would): each step is then one H2D copy, one call, one D2H copy
            prepared = [pkv.prepare_decode_step(
                dev_in["q"], dev_in["k_new"], dev_in["v_new"], dev_in["positions"],
                dev_in["slot_mapping"], copies[i]["k_cache"], copies[i]["v_cache"],
                dev_in["block_tables"], dev_in["decode_lens"], w.rope_theta, w.scale, outs[i],
                workspace=ws, partition_tokens=P_call, force_simt=args.simt, device_error=err)
                for i in range(ncopies)]

            def e2e_step(k):
                dbuf.copy_(hbuf, non_blocking=True)
                prepared[k % ncopies]()
                out_host.copy_(outs[k % ncopies], non_blocking=True)
        else:
            def e2e_step(k):
                c = dict(copies[k % ncopies], **dev_in)
                dbuf.copy_(hbuf, non_blocking=True)
                append(c)
                decode(c, outs[k % ncopies])
                out_host.copy_(outs[k % ncopies], non_blocking=True)

        Ke = max(1, min(K, 500))
        for k in range(3):
            e2e_step(k)
        e2e_ms = max_over_ranks(timed(Ke, e2e_step), world, device)
        e2e = {"value": round(world * nbytes / (e2e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
               "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}

    cpu = None
    if sample is not None:
        sub, frac = sample
        nthreads = os.cpu_count() or 1
        scales = (ks8, vs8) if e4m3 else None
        if e4m3:
            # the sample's packed 8-bit pages as the oracle's K and transposed V arrays
            k_h, v_h = W.e4m3_halves(sub.k_cache)
            sub.k_cache, sub.v_cache = k_h.contiguous(), v_h.contiguous()
        per_step, reps = time_oracle(sub, args.cpu_seconds, nthreads, scales, args.window)
        # the same oracle on one thread, briefly (reported beside the all-cores figure)
        per1, reps1 = time_oracle(sub, min(2.0, args.cpu_seconds), 1, scales, args.window)
        cpu = {"value": round(nbytes * frac / per_step / 1e9, 4), "unit": "GB/s",
               "cores": nthreads, "kind": "oracle",
               "value_1_thread": round(nbytes * frac / per1 / 1e9, 4),
               "sample": f"sequences 0..{len(sub.seqs) - 1} ({len(sub.seqs)} of {w.B}, "
                         f"{100 * frac:.1f} % of the step's K/V), one fp64 append + decode "
                         f"pass each, {reps} repetitions ({per_step * 1e3:.1f} ms each)"}

    block = dict(config_block(cfg, w, out_dtype, P, NP, args.simt, two_calls),
                 **({"sliding_window": args.window} if args.window else {}),
                 **({"step": "two calls (kv_append, paged_attention_decode_cascade over "
                             "the prefix groups)"} if cascade else {}),
                 l2=(f"inputs larger than L2 ({l2 >> 20} MiB): " +
                     (f"{ncopies} device-side copies of the per-layer tensors (q, new rows, "
                      f"K/V caches; the step's block tables, context lengths, positions "
                      f"and slots shared, as by the layers of a model); every timed step "
                      f"reads a copy that no step of the previous 2 x L2 bytes touched "
                      f"({nbytes / 1e6:.1f} MB read per step)" if ncopies > 1 else
                      f"the workload reads {nbytes / 1e6:.1f} MB per step") +
                     "; no flush inside the timed region"))
    traffic_key = (f"{cfg}_e4m3" if e4m3 else str(cfg)) if args.num_seqs is None else None
    res = {
        "value": round(value, 3), "unit": "GB/s", "steps": K, "warmup": Wu,
        "ms_per_step": round(step_ms_max, 5),
        "pct_of_hbm_peak": round(100.0 * value / (world * peak), 2),
        "seq_steps_per_s": round(world * w.B / (step_ms_max * 1e-3), 1),
        "dtype": "e4m3" if e4m3 else ("bf16" if w.dtype == torch.bfloat16 else "f32"),
        "config": block,
        "isolated_step": {"ms_per_step": round(iso_ms, 5),
                          "value": round(world * nbytes / (iso_ms * 1e-3) / 1e9, 3),
                          "ms_median": round(iso_each[len(iso_each) // 2], 5),
                          "ms_min": round(iso_each[0], 5), "ms_max": round(iso_each[-1], 5),
                          "how": "L2 flushed before each step, each step between its own "
                                 "pair of events"},
        "roofline": {"bound": "hbm",
                     "kernel": ("paged_attention_decode_cascade call: paged_decode_kernel + "
                                "cascade_prefix_kernel + combine_kernel") if cascade else
                               (("decode_step" if fused else "paged_attention_decode")
                                + " call: paged_decode_kernel" +
                                (" + combine_kernel" if kernels_per_decode == 2
                                 else (" (partitions merged in thread-block clusters)"
                                       if NP > 1 else ""))),
                     "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_src,
                     "decode_ms": round(decode_ms_max, 5),
                     "algorithmic_bytes": nbytes,
                     "traffic": recorded_traffic(traffic_key) if traffic_key else None},
        "gpu_launches": K * launches_per_step,
        "kv_append_us_per_call": round(append_ms * 1e3, 3),
        "clocks": clocks.summary(),
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    del copies, outs, w, ws
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, local)

    import paged_kv_cache_484_b200 as pkv
    pkv.load_library()
    cfg = args.config or HEADLINE_CONFIG
    head = measure(cfg, args, device, world, local, rank, full=True)
    per_config = None
    if args.config is None and not args.no_secondary:
        per_config = {}
        for c in SECONDARY_CONFIGS:
            r = measure(c, args, device, world, local, rank, full=False)
            per_config[r["config"]["workload"]] = {
                k: r[k] for k in ("value", "unit", "ms_per_step", "pct_of_hbm_peak",
                                  "seq_steps_per_s", "steps", "warmup", "roofline", "clocks",
                                  "isolated_step", "gpu_launches", "kv_append_us_per_call",
                                  "config")}
    line = {
        "metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world,
        "steps": head["steps"], "warmup": head["warmup"], "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": head["dtype"], "data": "synthetic",
        "pct_of_hbm_peak": head["pct_of_hbm_peak"], "seq_steps_per_s": head["seq_steps_per_s"],
        "config": head["config"], "isolated_step": head["isolated_step"],
        "roofline": head["roofline"],
        "gpu_launches": head["gpu_launches"] + sum(
            r["gpu_launches"] for r in (per_config or {}).values()),
        "kv_append_us_per_call": head["kv_append_us_per_call"],
        "clocks": head["clocks"], "e2e": head["e2e"], "cpu_baseline": head["cpu_baseline"],
        **({"per_config": per_config} if per_config is not None else {}),
        "device": torch.cuda.get_device_name(device),
        "versions": software_versions(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_prefill(args):
    """Chunked prefill on the workload's sequences: queries for the last C
    tokens of each context (their K/V are the cache's own rows), timed like
    the decode step: back to back from captured graphs over enough copies of
    the inputs to exceed L2.  Bytes: every context token's K and V once per
    kv head, plus q and out."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, local)
    import paged_kv_cache_484_b200 as pkv
    from paged_kv_cache_484_b200 import workloads as W

    pkv.load_library()
    cfg = args.config or 3
    w = W.make_config(cfg, device=device, num_seqs=args.num_seqs)
    if w.dtype != torch.bfloat16:
        raise SystemExit("prefill: bf16 workloads only")
    C = args.prefill
    lens = w.cached_lens.clamp(min=C).to(torch.int32)
    g = torch.Generator(device=device)
    g.manual_seed(484 + cfg)
    q = torch.randn((w.B, C, w.Hq, w.d), generator=g, device=device, dtype=torch.bfloat16)
    out_dtype = torch.bfloat16 if args.out_dtype == "bf16" else torch.float32
    P = args.partition_tokens or pkv.prefill_partition_tokens(w.B, C, w.Hq, w.Hkv, w.d,
                                                              w.max_blocks)
    need = pkv.prefill_workspace_size(w.B, C, w.Hq, w.Hkv, w.d, w.max_blocks,
                                      partition_tokens=P)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    esz_out = 2 if out_dtype == torch.bfloat16 else 4
    # K/V read per sequence: its whole context, or with a sliding window the
    # tokens from the chunk's first query's window on
    read = lens.to(torch.int64)
    if args.window:
        read = read.clamp(max=C - 1 + args.window)
    nbytes = int(read.sum().item()) * w.Hkv * w.d * 2 * 2 + w.B * C * w.Hq * w.d * (2 + esz_out)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    K = args.steps
    ncopies, S = copies_plan(nbytes, l2, K, args.copies)
    # per-layer q and caches copied; the block tables and lengths shared
    copies = [dict(q=q, k=w.k_cache, v=w.v_cache, t=w.block_tables, l=lens)]
    for _ in range(ncopies - 1):
        copies.append({k: (v.clone() if k in ("q", "k", "v") else v) for k, v in copies[0].items()})
    outs = [torch.empty((w.B, C, w.Hq, w.d), dtype=out_dtype, device=device)
            for _ in range(ncopies)]
    err = torch.zeros(1, dtype=torch.int32, device=device)

    def call(k):
        c = copies[k % ncopies]
        pkv.paged_attention_prefill(c["q"], c["k"], c["v"], c["t"], c["l"], w.scale,
                                    outs[k % ncopies], workspace=ws, partition_tokens=P,
                                    device_error=err, sliding_window=args.window)

    for k in range(max(3, args.warmup, ncopies)):
        call(k)
    torch.cuda.synchronize()

    def capture(n):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for k in range(n):
                call(k)
        return gr

    warm_order, timed_order = replay_order(K, S)
    graphs = {n: capture(n) for n in set(warm_order + timed_order)}
    for n in warm_order:
        graphs[n].replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        e0.record(stream)
        for n in timed_order:
            graphs[n].replay()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world, device)
    ms = max_over_ranks(e0.elapsed_time(e1) / K, world, device)
    if int(err.item()) != 0:
        raise SystemExit(f"device error flag {int(err.item()):#x}")
    peak, peak_src = load_peak()
    value = world * nbytes / (ms * 1e-3) / 1e9
    launches = 1 + (1 if -(-w.max_blocks * 16 // P) > 1 else 0)
    line = {
        "metric": "paged chunked-prefill attention achieved HBM GB/s; query tokens/sec",
        "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "query_tokens_per_s": round(world * w.B * C / (ms * 1e-3), 1),
        "config": {"workload": w.name + f"_prefill_chunk{C}",
                   "batch_seqs": w.B, "chunk_tokens": C, "q_heads": w.Hq, "kv_heads": w.Hkv,
                   **({"sliding_window": args.window} if args.window else {}),
                   "head_dim": w.d, "partition_tokens": P,
                   "l2": f"inputs larger than L2: {ncopies} copies, no flush in the timed region"},
        "roofline": {"bound": "hbm", "kernel": "paged_prefill_kernel" +
                     (" + prefill_combine_kernel" if launches == 2 else ""),
                     "achieved": round(value / world, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(value / world / peak, 4), "peak_source": peak_src,
                     "traffic": None},
        "gpu_launches": K * launches,
        "clocks": clocks.summary(),
        "device": torch.cuda.get_device_name(device),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.prefill:
        return run_prefill(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
