"""Helpers shared by the GPU parity tests.

The oracle never sees a value produced by the CUDA path: sub-problems are cut
from the workload's INPUT tensors (taken before the GPU step runs), then the
oracle performs its own append and decode on them.
"""
from __future__ import annotations

import math

import torch

import oracle
import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200.workloads import Workload, extract_sequences

TOL_F32 = 1e-5      # attention output, fp32 inputs
TOL_BF16 = 2e-3     # attention output, bf16 inputs (fp32 accumulation)


def ulp_bf16(x: torch.Tensor) -> torch.Tensor:
    """Spacing of bf16 numbers at |x| (x float64); subnormal spacing below 2^-126."""
    a = x.abs().clamp(min=2.0 ** -126)
    e = torch.floor(torch.log2(a))
    return torch.pow(2.0, e - 7)


class SubProblem:
    """Inputs of some sequences of a workload, copied to the host before the
    GPU step runs, and the oracle's own step on them."""

    def __init__(self, w: Workload, seqs):
        self.__dict__.update(vars(extract_sequences(w, seqs)))

    def oracle_step(self, nthreads=8, pairs=None, window=0):
        """Oracle append then decode (over the last ``window`` tokens when
        > 0); returns (q_rot, k_cache, v_cache, out_f64)."""
        q = self.q.clone()
        kc = self.k_cache.clone()
        vc = self.v_cache.clone()
        oracle.kv_append(q, self.k_new.clone(), self.v_new.clone(), self.positions, self.slots,
                         kc, vc, self.theta)
        out = oracle.paged_attention_decode(q, kc, vc, self.tables, self.decode_lens, self.scale,
                                            pairs=pairs, nthreads=nthreads, window=window)
        return q, kc, vc, out


def gpu_step(w: Workload, out_dtype=torch.float32, partition_tokens=0, force_simt=False,
             device_error=None, fused=False):
    """One decode step on the workload (in place): kv_append then
    paged_attention_decode, or the single-launch decode_step when ``fused``."""
    out = torch.empty((w.B, w.Hq, w.d), dtype=out_dtype, device=w.q.device)
    if fused:
        pkv.decode_step(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache, w.v_cache,
                        w.block_tables, w.decode_lens, w.rope_theta, w.scale, out,
                        partition_tokens=partition_tokens, force_simt=force_simt,
                        device_error=device_error)
        return out
    pkv.kv_append(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache, w.v_cache,
                  w.rope_theta, device_error=device_error)
    pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens, w.scale,
                               out, partition_tokens=partition_tokens, force_simt=force_simt,
                               device_error=device_error)
    return out


def check_decode(got: torch.Tensor, want: torch.Tensor, kv_dtype: torch.dtype, what=""):
    """Max-abs error bound: 1e-5 (fp32 inputs) or 2e-3 (bf16 inputs); a bf16
    output may add half a bf16 ulp of the exact value for its own rounding."""
    got = got.double().cpu()
    tol = torch.full_like(want, TOL_F32 if kv_dtype == torch.float32 else TOL_BF16)
    if got.dtype != want.dtype:
        pass
    err = (got - want).abs()
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    bad = err > tol
    assert not bad.any(), (f"{what}: max err {err.max().item():.3e} "
                           f"at {bad.nonzero()[0].tolist()} (tol {tol.max().item():.1e})")
    return err.max().item()


def check_decode_bf16_out(got: torch.Tensor, want: torch.Tensor, what=""):
    got = got.double().cpu()
    tol = TOL_BF16 + 0.5 * ulp_bf16(want.abs() + TOL_BF16)
    err = (got - want).abs()
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    bad = err > tol
    assert not bad.any(), f"{what}: max err {err.max().item():.3e} (bf16 out)"
    return err.max().item()


def check_within_one_bf16_ulp(got: torch.Tensor, want: torch.Tensor, what=""):
    """Appended/rotated values: |gpu - oracle| <= 1 bf16 ulp of the oracle value."""
    g = got.double().cpu()
    o = want.double().cpu()
    err = (g - o).abs()
    tol = ulp_bf16(o)
    bad = err > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} values off by more than 1 bf16 ulp"
    return (err / tol).max().item() if err.numel() else 0.0


def sample_pairs(w: Workload, seqs, n_heads_per_seq=4, seed=0):
    g = torch.Generator()
    g.manual_seed(seed)
    pairs = []
    for i, _ in enumerate(seqs):
        hs = torch.randperm(w.Hq, generator=g)[:n_heads_per_seq]
        for h in hs.tolist():
            pairs.append((i, h))
    return torch.tensor(pairs, dtype=torch.int64)


def scale_for(d):
    return 1.0 / math.sqrt(d)
