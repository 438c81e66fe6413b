"""Chunked prefill (multi-query attention over the paged cache) vs the fp64
oracle, through the C ABI (GPU only).

The chunk of each sequence is the last C tokens of its context; query i
attends to tokens 0 .. L - C + i.  The oracle computes each query as one
plain decode over that prefix.  Bar: max-abs error <= 2e-3 (bf16 inputs,
fp32 output), plus half a bf16 ulp when the output itself is bf16.
"""
from __future__ import annotations

import pytest
import torch

import oracle
import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200 import workloads as W
from tests.parity_util import TOL_BF16, ulp_bf16

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(lens, G, Hkv, d, C, seed):
    w = W.build_workload("prefill", lens, G * Hkv, Hkv, d, torch.bfloat16, 1e4, seed=seed,
                         device=DEV, pool_factor=1.2)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed + 1)
    q = torch.randn((w.B, C, w.Hq, d), generator=g, device=DEV, dtype=torch.bfloat16)
    lens_t = w.cached_lens.clone()
    return w, q, lens_t


def _oracle(w, q, lens_t):
    return oracle.paged_chunked_prefill(q.cpu(), w.k_cache.cpu(), w.v_cache.cpu(),
                                        w.block_tables.cpu(), lens_t.cpu(), w.scale, nthreads=8)


def _check(got, want, what, bf16_out=False):
    got = got.double().cpu()
    tol = torch.full_like(want, TOL_BF16)
    if bf16_out:
        tol = tol + 0.5 * ulp_bf16(want)
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    err = (got - want).abs()
    bad = err > tol
    assert not bad.any(), f"{what}: max err {err.max().item():.3e} at {bad.nonzero()[0].tolist()}"


@pytest.mark.parametrize("d,G", [(64, 1), (64, 4), (64, 8), (128, 2), (128, 4)])
@pytest.mark.parametrize("C", [1, 7, 16])
@pytest.mark.parametrize("P", [0, 64, 512])
def test_prefill_matches_oracle(d, G, C, P):
    lens = [300, 16, 1000, 47, 2049][: 3 if d == 128 else 5]
    lens = [max(L, C) for L in lens]
    w, q, lens_t = _case(lens, G, 2, d, C, seed=300 + d + G + C)
    out = torch.empty((w.B, C, w.Hq, d), dtype=torch.float32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.paged_attention_prefill(q, w.k_cache, w.v_cache, w.block_tables, lens_t, w.scale, out,
                                partition_tokens=P, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check(out, _oracle(w, q, lens_t), f"d{d} G{G} C{C} P{P}")


def test_prefill_many_row_groups_bf16_out():
    """C*G = 96 rows per kv head (three row groups), bf16 output."""
    w, q, lens_t = _case([900, 333], 4, 2, 64, 24, seed=41)
    out = torch.empty((w.B, 24, w.Hq, 64), dtype=torch.bfloat16, device=DEV)
    pkv.paged_attention_prefill(q, w.k_cache, w.v_cache, w.block_tables, lens_t, w.scale, out,
                                partition_tokens=128)
    torch.cuda.synchronize()
    _check(out, _oracle(w, q, lens_t), "row groups, bf16 out", bf16_out=True)


def test_prefill_whole_context_chunk_and_short_context():
    """A chunk as long as the context (the first prefill of a prompt); a
    context shorter than the chunk is flagged and its rows left untouched."""
    w, q, lens_t = _case([64, 40], 4, 2, 64, 40, seed=43)
    lens_t[0] = 40           # whole context is the chunk
    lens_t[1] = 39           # shorter than the chunk: invalid
    out = torch.full((w.B, 40, w.Hq, 64), 7.0, dtype=torch.float32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.paged_attention_prefill(q, w.k_cache, w.v_cache, w.block_tables, lens_t, w.scale, out,
                                partition_tokens=16, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv.DEVERR_CONTEXT_LEN
    want = _oracle(w, q[:1], lens_t[:1])
    sub = oracle.paged_chunked_prefill(q[:1].cpu(), w.k_cache.cpu(), w.v_cache.cpu(),
                                       w.block_tables[:1].cpu(), lens_t[:1].cpu(), w.scale)
    _check(out[:1], sub, "whole-context chunk")
    assert torch.equal(out[1].cpu(), torch.full_like(out[1].cpu(), 7.0))
    del want


def test_prefill_last_query_equals_decode():
    """The chunk's last query sees the whole context: the same numbers as
    the decode call up to rounding."""
    w, q, lens_t = _case([1500, 64, 700], 4, 8, 64, 8, seed=47)
    out = torch.empty((w.B, 8, w.Hq, 64), dtype=torch.float32, device=DEV)
    pkv.paged_attention_prefill(q, w.k_cache, w.v_cache, w.block_tables, lens_t, w.scale, out)
    dec = torch.empty((w.B, w.Hq, 64), dtype=torch.float32, device=DEV)
    pkv.paged_attention_decode(q[:, -1].contiguous(), w.k_cache, w.v_cache, w.block_tables,
                               lens_t, w.scale, dec)
    torch.cuda.synchronize()
    assert (out[:, -1] - dec).abs().max().item() < 1e-4


def test_prompt_chunks_then_decode_steps():
    """A small engine loop on one paged cache: a 40-token prompt appended and
    attended in two chunks (24 then 16 tokens), then three decode steps
    (fused append + decode), every output against the oracle running the same
    appends and attention on its own copy of the cache."""
    Hq, Hkv, d, bs = 8, 2, 64, 16
    B, NB, steps = 2, 16, 3
    total = 40 + steps
    g = torch.Generator()
    g.manual_seed(53)
    tables = torch.randperm(NB, generator=g)[: B * 4].view(B, 4).to(torch.int32)
    kc = torch.randn(NB, Hkv, bs, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, bs, d, generator=g).to(torch.bfloat16)
    q_all = torch.randn(B, total, Hq, d, generator=g).to(torch.bfloat16)
    k_all = torch.randn(B, total, Hkv, d, generator=g).to(torch.bfloat16)
    v_all = torch.randn(B, total, Hkv, d, generator=g).to(torch.bfloat16)
    theta, scale = 1e4, 1 / 8.0
    kc_g, vc_g, tables_g = kc.to(DEV), vc.to(DEV), tables.to(DEV)
    kc_o, vc_o = kc.clone(), vc.clone()

    def slots(pos):  # [B] int64 slot of each sequence's token at position pos
        return (tables[:, pos // bs].to(torch.int64) * bs + pos % bs)

    done = 0
    for C in (24, 16):
        pos = torch.arange(done, done + C, dtype=torch.int64)
        # append the chunk: T = B*C tokens
        q_tok = q_all[:, done:done + C].reshape(B * C, Hq, d).clone()
        k_tok = k_all[:, done:done + C].reshape(B * C, Hkv, d).clone()
        v_tok = v_all[:, done:done + C].reshape(B * C, Hkv, d).clone()
        positions = pos.repeat(B)
        slot = torch.stack([slots(p) for p in pos], 1).reshape(-1)
        q_g = q_tok.to(DEV)
        pkv.kv_append(q_g, k_tok.to(DEV), v_tok.to(DEV), positions.to(DEV), slot.to(DEV),
                      kc_g, vc_g, theta)
        q_o = q_tok.clone()
        oracle.kv_append(q_o, k_tok.clone(), v_tok.clone(), positions, slot, kc_o, vc_o, theta)
        done += C
        lens = torch.full((B,), done, dtype=torch.int32)
        out = torch.empty((B, C, Hq, d), dtype=torch.float32, device=DEV)
        pkv.paged_attention_prefill(q_g.view(B, C, Hq, d), kc_g, vc_g, tables_g, lens.to(DEV),
                                    scale, out, partition_tokens=16)
        torch.cuda.synchronize()
        want = oracle.paged_chunked_prefill(q_o.view(B, C, Hq, d), kc_o, vc_o, tables, lens,
                                            scale)
        _check(out, want, f"prompt chunk of {C}")
    for s in range(steps):
        pos = torch.full((B,), done, dtype=torch.int64)
        slot = slots(done)
        q_s, k_s, v_s = (t[:, done].clone() for t in (q_all, k_all, v_all))
        lens = torch.full((B,), done + 1, dtype=torch.int32)
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=DEV)
        pkv.decode_step(q_s.to(DEV), k_s.to(DEV), v_s.to(DEV), pos.to(DEV), slot.to(DEV), kc_g,
                        vc_g, tables_g, lens.to(DEV), theta, scale, out)
        torch.cuda.synchronize()
        q_o = q_s.clone()
        oracle.kv_append(q_o, k_s.clone(), v_s.clone(), pos, slot, kc_o, vc_o, theta)
        want = oracle.paged_attention_decode(q_o, kc_o, vc_o, tables, lens, scale)
        _check(out, want, f"decode step {s}")
        done += 1


@pytest.mark.parametrize("d,G,C,W,P", [
    (64, 4, 16, 1, 0), (64, 4, 16, 7, 64), (64, 4, 16, 40, 0), (64, 8, 7, 100, 64),
    (128, 4, 16, 33, 0), (64, 1, 1, 17, 16), (64, 4, 16, 5000, 0), (64, 4, 24, 16, 128),
])
def test_prefill_sliding_window(d, G, C, W, P):
    """Query i of the chunk attends to its last W tokens only.  Keys and
    values before the chunk's first window are NaN: reading one of them, or
    not masking it per row, shows up as a non-finite or wrong output."""
    lens = [300, 16, 1000, 47, 2049][: 3 if d == 128 else 5]
    lens = [max(L, C) for L in lens]
    w, q, lens_t = _case(lens, G, 2, d, C, seed=330 + d + G + C + W)
    want = oracle.paged_chunked_prefill(q.cpu(), w.k_cache.cpu(), w.v_cache.cpu(),
                                        w.block_tables.cpu(), lens_t.cpu(), w.scale, nthreads=8,
                                        window=W)
    tables = w.block_tables.cpu()
    for b, L in enumerate(lens_t.tolist()):
        t = torch.arange(max(0, L - C + 1 - W))   # no query of the chunk attends these
        blk = tables[b, t // 16].to(torch.int64).to(DEV)
        row = (t % 16).to(DEV)
        w.k_cache[blk, :, row] = float("nan")
        w.v_cache[blk, :, row] = float("nan")
    out = torch.empty((w.B, C, w.Hq, d), dtype=torch.float32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.paged_attention_prefill(q, w.k_cache, w.v_cache, w.block_tables, lens_t, w.scale, out,
                                partition_tokens=P, device_error=err, sliding_window=W)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check(out, want, f"window {W} d{d} G{G} C{C} P{P}")


def test_prefill_full_ragged_batch_sampled():
    """The chunked-prefill workload at full size (the ragged batch of 64
    sequences, 32/8 heads, d 64, C = 16, the library's partition length, as
    the benchmark times it: two CTAs per SM, longest contexts first), checked
    on the longest, a middle and the shortest context against the oracle run
    on just those sequences."""
    C = 16
    w = W.make_config(3, device=DEV)
    lens = w.cached_lens.clamp(min=C).to(torch.int32)
    g = torch.Generator(device=DEV)
    g.manual_seed(487)
    q = torch.randn((w.B, C, w.Hq, w.d), generator=g, device=DEV, dtype=torch.bfloat16)
    out = torch.empty((w.B, C, w.Hq, w.d), dtype=torch.float32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.paged_attention_prefill(q, w.k_cache, w.v_cache, w.block_tables, lens, w.scale, out,
                                device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    order = torch.argsort(lens.cpu(), descending=True).tolist()
    kc, vc = w.k_cache.cpu(), w.v_cache.cpu()
    for b in (order[0], order[len(order) // 2], order[-1]):
        want = oracle.paged_chunked_prefill(q[b:b + 1].cpu(), kc, vc,
                                            w.block_tables[b:b + 1].cpu(),
                                            lens[b:b + 1].cpu(), w.scale, nthreads=8)
        _check(out[b:b + 1], want, f"sequence {b} (context {int(lens[b])})")
