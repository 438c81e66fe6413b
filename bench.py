#!/usr/bin/env python3
"""Benchmark of one paged decode step: kv_append + paged_attention_decode.

Default workload: the Llama-3.2-1B-shaped single-layer decode step (batch 1,
32 query / 8 KV heads, head_dim 64, 2048 cached tokens + 1 appended, block
size 16, 4096-block shuffled pool, bf16).  ``--config N`` picks another of
the five named workloads.  Metric: achieved HBM GB/s of the step's
algorithmic bytes (K/V of every context token + q + out), with seq-steps/s
alongside.

Timing: W warm-up steps, then exactly K timed steps back to back between one
pair of CUDA events on the launch stream (synchronised on both sides); the
steps are replays of CUDA graphs that captured the library call(s) of
consecutive steps, so host-side marshalling does not set the pace.  The
inputs are larger than L2: when one copy of the workload touches less than
twice the L2 size per step, the bench holds enough device-side copies (like
the per-layer caches of a model) and step k runs on copy k mod n, so every
step reads its K/V from HBM.  ``isolated_step`` in the output is the older,
pessimistic figure: one step at a time, L2 flushed before it (512 MiB
written, then 256 MiB read so no dirty line remains), each step between its
own pair of events (whose own cost, a few microseconds, it includes).
Under torchrun every rank runs its own copy of the workload (weak scaling,
no collective on the data path); the step time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle on the same workload instead
(rank 0 only); it is the deliberately slow definition the CUDA path is
checked against, not an optimised baseline.
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
DEFAULT_CONFIG = 2


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--out-dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--partition-tokens", type=int, default=0)
    ap.add_argument("--copies", type=int, default=0,
                    help="device-side copies of the workload (0: enough to exceed L2)")
    ap.add_argument("--simt", action="store_true", help="bf16: CUDA-core decode kernel")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding window: each query attends to the last W tokens (two calls)")
    ap.add_argument("--kv-dtype", default="native", choices=["native", "e4m3"],
                    help="e4m3: the workload's cache as an 8-bit cache (per-tensor scales), "
                         "stepped as kv_append_e4m3 + paged_attention_decode_e4m3")
    ap.add_argument("--two-calls", action="store_true",
                    help="time kv_append + paged_attention_decode as two launches instead of "
                         "the single-launch decode_step")
    ap.add_argument("--cascade", action="store_true",
                    help="two calls, the decode as paged_attention_decode_cascade over the "
                         "workload's prefix groups (config 4)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
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


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_484_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def software_versions() -> dict:
    """Versions the numbers were taken with (NVML read only)."""
    v = {"torch": torch.__version__, "cuda_runtime": torch.version.cuda,
         "kernel_sources": kernel_source_hash()}
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
    taken on the current kernel sources (else None).  ``cfg``: the config
    number, or e.g. "3_e4m3" for its 8-bit cache."""
    path = os.path.join(ROOT, "profiles", "decode_dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    ent = rec.get("configs", {}).get(str(cfg))
    return None if ent is None else ent.get("bytes_per_launch")


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML (read only) while the
    timed region runs."""

    REASONS = {
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
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

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
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
    if w.k_cache.dtype == torch.uint8:
        return {
            "workload": W.CONFIG_NAMES[cfg] + "_e4m3cache",
            "batch_seqs": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d,
            "context": s["ctx"], "tokens_decoded": int(w.decode_lens.to(torch.int64).sum().item()),
            "block_size": w.block_size, "pool_blocks": w.num_blocks,
            "kv_dtype": "e4m3 (per-tensor scales: max|x| / 448)",
            "kv_scales": list(w.meta.get("e4m3_scales", ())),
            "out_dtype": "bf16" if out_dtype == torch.bfloat16 else "f32",
            "partition_tokens": P, "max_partitions": NP, "decode_kernel": "mma_f16 (e4m3 pages)",
            "step": "two calls (kv_append_e4m3, paged_attention_decode_e4m3)",
        }
    return {
        "workload": W.CONFIG_NAMES[cfg],
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


# ---------------------------------------------------------------- oracle arm

def time_oracle(w, seconds: float, nthreads: int, e4m3_scales=None, window: int = 0):
    """Oracle append + decode of the whole workload (or a bounded subset of
    sequences for the big ones), repeated until ~``seconds`` of CPU time
    (the 8-bit cache's append and decode when ``e4m3_scales`` is given)."""
    import oracle
    from paged_kv_cache_484_b200.workloads import extract_sequences

    order = list(range(w.B))
    # bounded sample: whole sequences until the sample holds <= 8M context tokens
    lens = w.decode_lens.cpu().tolist()
    seqs, tok = [], 0
    for b in order:
        if seqs and tok + lens[b] > 8_000_000:
            break
        seqs.append(b)
        tok += lens[b]
    sub = extract_sequences(w, seqs)
    att = [min(L, window) if window else L for L in lens]  # attended tokens
    frac_bytes = sum(att[b] for b in seqs) / max(1, sum(att))
    reps, t_total = 0, 0.0
    while t_total < seconds or reps == 0:
        q = sub.q.clone()
        kc, vc = sub.k_cache.clone(), sub.v_cache.clone()
        t0 = time.perf_counter()
        if e4m3_scales is not None:
            ks, vs = e4m3_scales
            oracle.kv_append_e4m3(q, sub.k_new.clone(), sub.v_new.clone(), sub.positions,
                                  sub.slots, kc, vc, sub.theta, ks, vs)
            oracle.paged_attention_decode_e4m3(q, kc, vc, sub.tables, sub.decode_lens, sub.scale,
                                               ks, vs, nthreads=nthreads, window=window)
        else:
            oracle.kv_append(q, sub.k_new.clone(), sub.v_new.clone(), sub.positions, sub.slots,
                             kc, vc, sub.theta)
            oracle.paged_attention_decode(q, kc, vc, sub.tables, sub.decode_lens, sub.scale,
                                          nthreads=nthreads, window=window)
        t_total += time.perf_counter() - t0
        reps += 1
    return t_total / reps, seqs, frac_bytes, reps


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    from paged_kv_cache_484_b200 import workloads as W
    out_dtype = torch.bfloat16 if args.out_dtype == "bf16" else torch.float32
    w = W.make_config(args.config, device="cpu")
    nthreads = os.cpu_count() or 1
    per_step, seqs, frac, reps = time_oracle(w, max(1.0, min(args.cpu_seconds, 60.0)), nthreads)
    bytes_sample = step_bytes(w, out_dtype) * frac
    value = bytes_sample / per_step / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": reps, "warmup": 0,
        "ms_per_step": round(per_step * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "seq_steps_per_s": round(len(seqs) / per_step, 3),
        "config": config_block(args.config, w, out_dtype, None, None, False),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": nthreads,
                         "kind": "oracle",
                         "sample": f"{len(seqs)} of {w.B} sequences, full append+decode step, "
                                   f"{reps} repetitions"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- CUDA arm

def run_ours(args):
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, local)

    import paged_kv_cache_484_b200 as pkv
    from paged_kv_cache_484_b200 import workloads as W

    pkv.load_library()
    out_dtype = torch.bfloat16 if args.out_dtype == "bf16" else torch.float32
    w = W.make_config(args.config, device=device)
    e4m3 = args.kv_dtype == "e4m3"
    if e4m3:
        if w.dtype != torch.bfloat16:
            raise SystemExit("--kv-dtype e4m3 takes a bf16 workload (configs 2-5)")
        k8, v8, ks8, vs8 = W.e4m3_cache(w)
        w.k_cache, w.v_cache = k8, v8
        w.meta["e4m3_scales"] = (ks8, vs8)
        args.two_calls = True
        torch.cuda.empty_cache()
    kv_dt = torch.uint8 if e4m3 else w.dtype
    host_inputs = None
    if not args.no_e2e:
        # pristine copies of the per-step inputs, in pinned host memory
        host_inputs = {k: v.cpu().pin_memory() for k, v in dict(
            q=w.q, k_new=w.k_new, v_new=w.v_new, positions=w.positions,
            slot_mapping=w.slot_mapping, block_tables=w.block_tables,
            decode_lens=w.decode_lens).items()}

    P = args.partition_tokens or pkv.decode_partition_tokens(w.B, w.Hq, w.Hkv, w.d, w.max_blocks,
                                                              kv_dtype=kv_dt)
    NP = math.ceil(w.max_blocks * w.block_size / P)
    ws_bytes = pkv.decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks, kv_dtype=kv_dt,
                                         partition_tokens=P)
    ws = pkv.new_workspace(ws_bytes, device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    nbytes = step_bytes(w, out_dtype, args.window)
    if args.window:
        if args.cascade:
            raise SystemExit("--window and --cascade do not combine")
        args.two_calls = True

    # Inputs larger than L2: device-side copies of the workload (every tensor
    # a step reads or writes), step k on copy k mod n.
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    ncopies = 1 if nbytes >= 2 * l2 else min(1024, math.ceil(2 * l2 / nbytes))
    if args.copies:
        ncopies = args.copies
    # Per-layer tensors (q, the new rows, the caches) get their own copy; the
    # step's metadata (positions, slots, block tables, context lengths) is one
    # set shared by all copies, as one decode step's metadata is shared by all
    # layers of a model.
    layer_fields = ("q", "k_new", "v_new", "k_cache", "v_cache")
    step_fields = ("positions", "slot_mapping", "block_tables", "decode_lens")
    copies = [dict((f, getattr(w, f)) for f in layer_fields + step_fields)]
    for _ in range(ncopies - 1):
        copies.append(dict([(f, getattr(w, f).clone()) for f in layer_fields] +
                           [(f, getattr(w, f)) for f in step_fields]))
    outs = [torch.empty((w.B, w.Hq, w.d), dtype=out_dtype, device=device) for _ in range(ncopies)]

    cascade = args.cascade
    if cascade:
        if e4m3:
            raise SystemExit("--cascade takes the bf16 cache")
        if w.meta.get("prefix_group", 0) <= 1:
            raise SystemExit("--cascade needs a workload with prefix groups (config 4)")
        args.two_calls = True
        grp = int(w.meta["prefix_group"])
        group_start = torch.tensor(list(range(0, w.B, grp)) + [w.B], dtype=torch.int32,
                                   device=device)
        cached = w.cached_lens.to(torch.int64)
        shared_tokens = (torch.minimum(cached // 16,
                                       torch.full_like(cached, w.meta["prefix_tokens"] // 16))
                         * 16).to(torch.int32)
        ws = pkv.new_workspace(pkv.decode_cascade_workspace_size(
            w.B, w.Hq, w.Hkv, w.d, w.max_blocks, partition_tokens=P), device)
    fused = not args.two_calls
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
        if e4m3:
            pkv.kv_append_e4m3(c["q"], c["k_new"], c["v_new"], c["positions"], c["slot_mapping"],
                               c["k_cache"], c["v_cache"], w.rope_theta, ks8, vs8,
                               device_error=err)
        elif not fused:
            pkv.kv_append(c["q"], c["k_new"], c["v_new"], c["positions"], c["slot_mapping"],
                          c["k_cache"], c["v_cache"], w.rope_theta, device_error=err)

    def decode(c, out):
        if e4m3:
            pkv.paged_attention_decode_e4m3(c["q"], c["k_cache"], c["v_cache"],
                                            c["block_tables"], c["decode_lens"], w.scale, ks8,
                                            vs8, out, workspace=ws, partition_tokens=P,
                                            device_error=err, sliding_window=args.window)
        elif fused:
            pkv.decode_step(c["q"], c["k_new"], c["v_new"], c["positions"], c["slot_mapping"],
                            c["k_cache"], c["v_cache"], c["block_tables"], c["decode_lens"],
                            w.rope_theta, w.scale, out, workspace=ws, partition_tokens=P,
                            force_simt=args.simt, device_error=err)
        elif cascade:
            pkv.paged_attention_decode_cascade(c["q"], c["k_cache"], c["v_cache"],
                                               c["block_tables"], c["decode_lens"], group_start,
                                               shared_tokens, grp, w.scale, out, workspace=ws,
                                               partition_tokens=P, force_simt=args.simt,
                                               device_error=err)
        else:
            pkv.paged_attention_decode(c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                                       c["decode_lens"], w.scale, out, workspace=ws,
                                       partition_tokens=P, force_simt=args.simt,
                                       device_error=err, sliding_window=args.window)

    def step(k):
        c = copies[k % ncopies]
        append(c)
        decode(c, outs[k % ncopies])

    stream = torch.cuda.current_stream(device)
    Wu = max(3, args.warmup)
    for k in range(max(Wu, ncopies)):
        step(k)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"device error flag {int(err.item()):#x} during warm-up")

    def timed(K, body):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier(world, device)
        torch.cuda.synchronize()
        e0.record(stream)
        for k in range(K):
            body(k)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world, device)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K

    # The timed steps are replays of CUDA graphs that captured S consecutive
    # steps (steps 0..S-1, one per copy when there are copies), launches and
    # programmatic dependencies as the library issues them: the host's
    # per-call marshalling (tens of microseconds in Python) then does not set
    # the pace of a step whose kernels take a few microseconds, and the next
    # step's decode launches while the current one ends, as consecutive
    # layers would.  K = q S + r steps are q replays of the S-step graph and
    # one of an r-step graph.
    K = args.steps
    S = ncopies if ncopies > 1 else min(K, 16)

    def capture(body, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for k in range(n):
                body(k)
        return g

    def graphs_for(body):
        full = capture(body, S)
        tail = capture(body, K % S) if K % S else None
        torch.cuda.synchronize()
        return full, tail

    def replay(gt):
        def run(_):
            for _ in range(K // S):
                gt[0].replay()
            if gt[1] is not None:
                gt[1].replay()
        return run

    step_g = graphs_for(step)
    decode_g = step_g if fused else graphs_for(lambda k: decode(copies[k % ncopies],
                                                                outs[k % ncopies]))
    for _ in range(max(1, -(-Wu // S))):
        step_g[0].replay()
    torch.cuda.synchronize()

    # kv_append alone (not part of the roofline claim): the same graphs-of-S
    # scheme over the copies
    def append_only(k):
        c = copies[k % ncopies]
        if e4m3:
            append(c)
        else:
            pkv.kv_append(c["q"], c["k_new"], c["v_new"], c["positions"], c["slot_mapping"],
                          c["k_cache"], c["v_cache"], w.rope_theta, device_error=err)

    append_g = graphs_for(append_only)

    with ClockSampler(local) as clocks:
        step_ms = timed(1, replay(step_g)) / K
        # the decode call alone (the same call as the step when it is fused)
        decode_ms = step_ms if fused else timed(1, replay(decode_g)) / K
    append_ms = max_over_ranks(timed(1, replay(append_g)) / K, world, device)
    step_ms_max = max_over_ranks(step_ms, world, device)
    decode_ms_max = max_over_ranks(decode_ms, world, device)
    if int(err.item()) != 0:
        raise SystemExit(f"device error flag {int(err.item()):#x} during timing")

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
                workspace=ws, partition_tokens=P, force_simt=args.simt, device_error=err)
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
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wc = W.make_config(args.config, device="cpu") if args.config in (1, 2, 3) else None
        if wc is None:
            # big workloads: the oracle reads a bounded subset copied from the device
            wc = w
        nthreads = os.cpu_count() or 1
        if e4m3 and wc is not w:
            k8c, v8c, _, _ = W.e4m3_cache(wc)
            wc.k_cache, wc.v_cache = k8c, v8c
        per_step, seqs, frac, reps = time_oracle(wc, args.cpu_seconds, nthreads,
                                                 (ks8, vs8) if e4m3 else None, args.window)
        # the same oracle on one thread, briefly (reported beside the all-cores figure)
        per1, seqs1, frac1, reps1 = time_oracle(wc, min(2.0, args.cpu_seconds), 1,
                                                (ks8, vs8) if e4m3 else None, args.window)
        cpu = {"value": round(nbytes * frac / per_step / 1e9, 4), "unit": "GB/s",
               "cores": nthreads, "kind": "oracle",
               "value_1_thread": round(nbytes * frac1 / per1 / 1e9, 4),
               "sample": f"{len(seqs)} of {w.B} sequences, full append+decode step in fp64, "
                         f"{reps} repetitions ({per_step * 1e3:.1f} ms each)"}

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": max(3, args.warmup), "ms_per_step": round(step_ms_max, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if e4m3 else ("bf16" if w.dtype == torch.bfloat16 else "f32"),
        "data": "synthetic",
        "pct_of_hbm_peak": round(100.0 * value / (world * peak), 2),
        "seq_steps_per_s": round(world * w.B / (step_ms_max * 1e-3), 1),
        "config": dict(config_block(args.config, w, out_dtype, P, NP, args.simt, args.two_calls),
                       **({"sliding_window": args.window} if args.window else {}),
                       **({"step": "two calls (kv_append, paged_attention_decode_cascade over "
                                   "the prefix groups)"} if cascade else {}),
                       l2=(f"inputs larger than L2 ({l2 >> 20} MiB): " +
                           (f"{ncopies} device-side copies of the per-layer tensors (q, new rows, "
                            f"K/V caches; the step's block tables, context lengths, positions "
                            f"and slots shared, as by the layers of a model), step k on copy k "
                            f"mod {ncopies} ({nbytes / 1e6:.1f} MB read per step)" if ncopies > 1 else
                            f"the workload reads {nbytes / 1e6:.1f} MB per step") +
                           "; no flush inside the timed region")),
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
                     "traffic": recorded_traffic(f"{args.config}_e4m3" if e4m3 else args.config)},
        "gpu_launches": K * launches_per_step,
        "kv_append_us_per_call": round(append_ms * 1e3, 3),
        "clocks": clocks.summary(),
        "e2e": e2e,
        "cpu_baseline": cpu,
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
    w = W.make_config(args.config, device=device)
    if w.dtype != torch.bfloat16:
        raise SystemExit("prefill: bf16 workloads only")
    C = args.prefill
    lens = w.cached_lens.clamp(min=C).to(torch.int32)
    g = torch.Generator(device=device)
    g.manual_seed(484 + args.config)
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
    ncopies = args.copies or (1 if nbytes >= 2 * l2 else min(1024, math.ceil(2 * l2 / nbytes)))
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
    K = args.steps
    S = ncopies if ncopies > 1 else min(K, 16)

    def capture(n):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for k in range(n):
                call(k)
        return gr

    full = capture(S)
    tail = capture(K % S) if K % S else None
    full.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        e0.record(stream)
        for _ in range(K // S):
            full.replay()
        if tail is not None:
            tail.replay()
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
        "config": {"workload": W.CONFIG_NAMES[args.config] + f"_prefill_chunk{C}",
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
