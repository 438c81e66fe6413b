"""Approximate quality of the 8-bit cache, kept apart from exact execution
("Efficient LLM Inference", Verify Exact Execution and Approximate Quality
Separately).  CPU only, oracle only: the GPU parity tests check the kernels
against the oracle on the same codes; this file says what the format itself
costs against the bf16 cache.

* Values already on the E4M3 grid (times a power-of-two scale) lose nothing:
  the 8-bit decode equals the bf16-cache decode up to fp64 rounding.
* N(0, 1) K/V with 1 % of the key rows x8 (the long-context workload's
  peaked keys), per-tensor scales max|x| / 448: the output moves by a few
  percent of its RMS -- E4M3 keeps 3 mantissa bits, a relative rounding
  error of at most 2^-4 per element.  The bound asserted is loose; the
  measured figures are printed with -s.
"""
from __future__ import annotations

import torch

import oracle
from paged_kv_cache_484_b200 import workloads as W


def _workload(seed, hot):
    lens = [300, 2049, 17, 1000, 4000, 64]
    return W.build_workload("quality", [L - 1 for L in lens], 32, 8, 64, torch.bfloat16, 5e5,
                            seed, "cpu", pool_factor=1.1, hot_key_frac=hot)


def test_values_on_the_grid_are_kept_exactly():
    w = _workload(71, 0.0)
    g = torch.Generator().manual_seed(72)
    codes = {}
    # the caches become E4M3 values x 2^-4 (exact in bf16), with 28 = 448 x 2^-4
    # present so that the per-tensor scale max|x| / 448 is exactly 2^-4
    for name in ("k_cache", "v_cache"):
        c = torch.randint(0, 256, getattr(w, name).shape, generator=g, dtype=torch.int32)
        c = torch.where((c & 0x7F) >= 0x7F, c & 0x80, c).to(torch.uint8)
        c[0, 0, 0, 0] = 0x7E
        codes[name] = c
        setattr(w, name, (c.view(torch.float8_e4m3fn).to(torch.float32) * 2.0 ** -4)
                .to(torch.bfloat16))
    k8, v8, ks, vs = W.e4m3_cache(w)
    assert ks == vs == 2.0 ** -4
    assert torch.equal(k8, codes["k_cache"])
    assert torch.equal(v8, codes["v_cache"].transpose(2, 3))
    ref = oracle.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                        w.scale, nthreads=8)
    got = oracle.paged_attention_decode_e4m3(w.q, k8, v8, w.block_tables, w.decode_lens, w.scale,
                                             ks, vs, nthreads=8)
    assert (got - ref).abs().max().item() < 1e-12


def test_quantization_error_of_normal_caches():
    w = _workload(73, 0.01)
    k8, v8, ks, vs = W.e4m3_cache(w)
    ref = oracle.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                        w.scale, nthreads=8)
    got = oracle.paged_attention_decode_e4m3(w.q, k8, v8, w.block_tables, w.decode_lens, w.scale,
                                             ks, vs, nthreads=8)
    err = got - ref
    rel_rms = (err.pow(2).mean().sqrt() / ref.pow(2).mean().sqrt()).item()
    print(f"\n8-bit cache vs bf16 cache: k_scale {ks:.4g}, v_scale {vs:.4g}, "
          f"max abs err {err.abs().max().item():.3f}, relative RMS err {rel_rms:.4f}")
    assert torch.isfinite(got).all()
    assert rel_rms < 0.1
