"""The 8-bit (E4M3) cache through the C ABI vs the fp64 oracle (GPU only).

Exact execution and approximate quality are checked separately, as
"Efficient LLM Inference" asks of quantized outputs:
  * exact: the append's codes are bit-identical to the oracle's (the same
    binary32 decision, then nearest E4M3); the decode over a given 8-bit
    cache matches the oracle's fp64 decode over the same codes within the
    bf16-input bound, 2e-3;
  * approximate: how far the 8-bit cache moves the attention output from the
    bf16 cache is a property of the format, reported in
    test_e4m3_quality.py (CPU, oracle only), not a parity bar.

Unused rows of the pool hold random bytes, NaN codes included, so the tests
also show that no byte outside a sequence's context reaches its output.
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200.workloads import e4m3_halves, e4m3_pack
from tests.parity_util import TOL_BF16, ulp_bf16

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
BS = 16


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def _codes(shape, g, sigma=16.0):
    """E4M3 codes of N(0, sigma^2) draws (PyTorch's float8 cast)."""
    x = (torch.randn(shape, generator=g) * sigma).clamp(-448.0, 448.0)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def _cache(lens, Hkv, d, seed, peaked=0.01):
    """Paged 8-bit pool: every byte random first, then each sequence's tokens
    written as codes of N(0, 16^2) (a fraction `peaked` of the key rows x8)."""
    g = _gen(seed)
    need = [max(1, math.ceil(L / BS)) for L in lens]
    NB = int(sum(need) * 1.3) + 2
    perm = torch.randperm(NB, generator=g)
    tables = torch.full((len(lens), max(need)), -1, dtype=torch.int32)
    kc = torch.randint(0, 256, (NB, Hkv, BS, d), generator=g, dtype=torch.int32).to(torch.uint8)
    vc = torch.randint(0, 256, (NB, Hkv, d, BS), generator=g, dtype=torch.int32).to(torch.uint8)
    c = 0
    for b, L in enumerate(lens):
        ids = perm[c:c + need[b]]
        c += need[b]
        tables[b, :need[b]] = ids.to(torch.int32)
        if L == 0:
            continue
        t = torch.arange(L)
        blk, row = ids[t // BS], t % BS
        sig = torch.where(torch.rand(L, generator=g) < peaked, 128.0, 16.0)
        K = (torch.randn(L, Hkv, d, generator=g) * sig[:, None, None]).clamp(-448.0, 448.0)
        K = K.to(torch.float8_e4m3fn).view(torch.uint8)
        V = _codes((L, Hkv, d), g)
        kc[blk, :, row, :] = K
        vc[blk, :, :, row] = V
    return kc, vc, tables


def _check(got, want, what, out_dtype=torch.float32):
    got = got.double().cpu()
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    tol = TOL_BF16 + (0.5 * ulp_bf16(want) if out_dtype == torch.bfloat16 else 0.0)
    err = (got - want).abs() - tol
    assert err.max().item() <= 0.0, f"{what}: max err over bound {err.max().item():.3e}"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d", [64, 128])
def test_kv_append_e4m3_codes_bit_exact(dtype, d):
    g = _gen(500 + d)
    T, Hq, Hkv, NB = 7, 16, 4, 12
    q = torch.randn(T, Hq, d, generator=g).to(dtype)
    k = (torch.randn(T, Hkv, d, generator=g) * 3).to(dtype)
    v = (torch.randn(T, Hkv, d, generator=g) * 3).to(dtype)
    k[2, 0, :4] = 1e4  # saturates
    pos = torch.tensor([0, 5, 17, 300, 4095, 131071, 9], dtype=torch.int64)
    slots = torch.tensor([3, 16 * 4 + 15, -1, 17, 16 * 11, 100, 16 * 7 + 8], dtype=torch.int64)
    ks, vs = 0.0173, 0.0291
    kc = torch.full((NB, Hkv, BS, d), 0x7F, dtype=torch.uint8)
    vc = torch.full((NB, Hkv, d, BS), 0x7F, dtype=torch.uint8)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    qg, kvg = q.to(DEV), e4m3_pack(kc, vc).to(DEV)
    pkv.kv_append_e4m3(qg, k.to(DEV), v.to(DEV), pos.to(DEV), slots.to(DEV), kvg, 5e5, ks,
                       vs, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    qo = q.clone()
    oracle.kv_append_e4m3(qo, k.clone(), v.clone(), pos, slots, kc, vc, 5e5, ks, vs)
    kcg, vcg = (h.cpu() for h in e4m3_halves(kvg))
    assert torch.equal(kcg, kc), f"k codes differ at {(kcg != kc).nonzero()[:4].tolist()}"
    assert torch.equal(vcg, vc), f"v codes differ at {(vcg != vc).nonzero()[:4].tolist()}"
    dq = (qg.cpu().double() - qo.double()).abs()
    bound = ulp_bf16(qo.double()) if dtype == torch.bfloat16 else 1e-6 * qo.double().abs() + 1e-30
    assert (dq <= bound).all(), "rotated q"


def test_kv_append_e4m3_slot_out_of_range():
    T, Hq, Hkv, d, NB = 2, 8, 2, 64, 4
    q = torch.randn(T, Hq, d, device=DEV).to(torch.bfloat16)
    k = torch.randn(T, Hkv, d, device=DEV).to(torch.bfloat16)
    kv = torch.zeros(NB, Hkv, 2, BS * d, dtype=torch.uint8, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    slots = torch.tensor([NB * BS, 5], dtype=torch.int64, device=DEV)
    pos = torch.tensor([1, 2], dtype=torch.int64, device=DEV)
    pkv.kv_append_e4m3(q, k, k.clone(), pos, slots, kv, 1e4, 0.05, 0.05, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv.DEVERR_SLOT
    kc, vc = e4m3_halves(kv)
    assert kc[0, :, 5].any() and vc[0, :, :, 5].any() and not kv[1:].any()


@pytest.mark.parametrize("d,G,P,cluster", [
    (64, 4, 0, True), (64, 4, 64, True), (64, 4, 64, False), (64, 4, 16, False),
    (64, 1, 0, True), (64, 2, 128, False), (64, 8, 0, True), (64, 8, 48, False),
    (128, 4, 0, True), (128, 4, 256, False), (128, 8, 0, True), (128, 1, 64, True),
    (128, 8, 16, False),  # merge rows in a region of their own, many one-page items
])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_e4m3_matches_oracle(d, G, P, cluster, out_dtype):
    lens = [1, 15, 16, 17, 300, 2049, 64, 0, 5, 1000]
    Hkv = 2
    kc, vc, tables = _cache(lens, Hkv, d, seed=600 + d + G + P)
    B = len(lens)
    q = torch.randn(B, Hkv * G, d, generator=_gen(601 + G)).to(torch.bfloat16)
    cl = torch.tensor(lens, dtype=torch.int32)
    ks, vs, scale = 1 / 16, 1 / 16, 1 / math.sqrt(d)
    out = torch.empty(B, Hkv * G, d, dtype=out_dtype, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.paged_attention_decode_e4m3(q.to(DEV), e4m3_pack(kc, vc).to(DEV), tables.to(DEV),
                                    cl.to(DEV), scale, ks, vs, out, partition_tokens=P,
                                    cluster=cluster, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle.paged_attention_decode_e4m3(q, kc, vc, tables, cl, scale, ks, vs, nthreads=8)
    _check(out, want, f"e4m3 d{d} G{G} P{P} cluster{cluster}", out_dtype)


def test_decode_e4m3_cluster_modes_agree():
    """Batch 1 at 2048 tokens: the cluster merge and the combine kernel give
    the same result within rounding, and both match the oracle."""
    lens, Hkv, d, G = [2049], 8, 64, 4
    kc, vc, tables = _cache(lens, Hkv, d, seed=610)
    q = torch.randn(1, Hkv * G, d, generator=_gen(611)).to(torch.bfloat16)
    cl = torch.tensor(lens, dtype=torch.int32)
    args = [t.to(DEV) for t in (q, e4m3_pack(kc, vc), tables, cl)]
    outs = []
    for cluster in (True, False):
        out = torch.empty(1, Hkv * G, d, dtype=torch.float32, device=DEV)
        pkv.paged_attention_decode_e4m3(*args, 0.125, 0.05, 0.07, out, cluster=cluster)
        outs.append(out)
    torch.cuda.synchronize()
    want = oracle.paged_attention_decode_e4m3(q, kc, vc, tables, cl, 0.125, 0.05, 0.07)
    for o in outs:
        _check(o, want, "batch 1")
    assert (outs[0] - outs[1]).abs().max().item() < 1e-4


def test_e4m3_append_then_decode_ragged_batch():
    """The two-call step on a ragged batch shaped like the 64-sequence
    workload (contexts U[128, 4096], 32/8 heads, d 64): append one new token
    per sequence into the 8-bit cache, then decode over L + 1 tokens, at the
    partition length the library picks; against the oracle doing the same."""
    g = _gen(620)
    B, Hkv, G, d = 64, 8, 4, 64
    lens = torch.randint(128, 4097, (B,), generator=g).tolist()
    kc, vc, tables = _cache([L + 1 for L in lens], Hkv, d, seed=621)
    q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
    pos = torch.tensor(lens, dtype=torch.int64)
    slots = torch.tensor([int(tables[b, L // BS]) * BS + L % BS for b, L in enumerate(lens)],
                         dtype=torch.int64)
    cl = torch.tensor([L + 1 for L in lens], dtype=torch.int32)
    ks, vs, theta, scale = 1 / 16, 1 / 16, 5e5, 0.125
    qg, kvg = q.to(DEV), e4m3_pack(kc, vc).to(DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.kv_append_e4m3(qg, kn.to(DEV), vn.to(DEV), pos.to(DEV), slots.to(DEV), kvg, theta,
                       ks, vs, device_error=err)
    out = torch.empty(B, Hkv * G, d, dtype=torch.float32, device=DEV)
    pkv.paged_attention_decode_e4m3(qg, kvg, tables.to(DEV), cl.to(DEV), scale, ks, vs, out,
                                    device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    qo, kco, vco = q.clone(), kc.clone(), vc.clone()
    oracle.kv_append_e4m3(qo, kn.clone(), vn.clone(), pos, slots, kco, vco, theta, ks, vs)
    kcg, vcg = (h.cpu() for h in e4m3_halves(kvg))
    assert torch.equal(kcg, kco) and torch.equal(vcg, vco), "appended codes"
    want = oracle.paged_attention_decode_e4m3(qo, kco, vco, tables, cl, scale, ks, vs, nthreads=16)
    _check(out, want, "ragged batch step")


def _step_case(lens, Hkv, G, d, seed):
    """Inputs of one decode step over the 8-bit cache: context lens[b]
    includes the new token L - 1, whose slot is the one the table gives it."""
    kc, vc, tables = _cache(lens, Hkv, d, seed=seed)
    g = _gen(seed + 1)
    B = len(lens)
    q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16)
    kn = (torch.randn(B, Hkv, d, generator=g) * 1.5).to(torch.bfloat16)
    vn = (torch.randn(B, Hkv, d, generator=g) * 1.5).to(torch.bfloat16)
    pos = torch.tensor([max(L - 1, 0) + 7 * b for b, L in enumerate(lens)], dtype=torch.int64)
    slots = torch.tensor([int(tables[b, (L - 1) // BS]) * BS + (L - 1) % BS if L > 0 else -1
                          for b, L in enumerate(lens)], dtype=torch.int64)
    cl = torch.tensor(lens, dtype=torch.int32)
    return kc, vc, tables, q, kn, vn, pos, slots, cl


def _oracle_step(kc, vc, tables, q, kn, vn, pos, slots, cl, theta, scale, ks, vs, window=0):
    qo, kco, vco = q.clone(), kc.clone(), vc.clone()
    oracle.kv_append_e4m3(qo, kn.clone(), vn.clone(), pos, slots, kco, vco, theta, ks, vs)
    if window:
        want = oracle.paged_attention_decode_e4m3(qo, kco, vco, tables, cl, scale, ks, vs,
                                                  nthreads=8, window=window)
    else:
        want = oracle.paged_attention_decode_e4m3(qo, kco, vco, tables, cl, scale, ks, vs,
                                                  nthreads=8)
    return kco, vco, want


@pytest.mark.parametrize("d,G,P,cluster", [
    (64, 4, 0, True), (64, 4, 64, False), (64, 1, 16, False), (64, 8, 0, True),
    (64, 2, 128, False), (128, 4, 0, True), (128, 8, 48, False), (128, 1, 0, True),
    (128, 2, 256, False),
])
def test_decode_step_e4m3_matches_oracle(d, G, P, cluster):
    """The one-launch step: the new codes in the cache equal the oracle
    append's bit for bit, q is left as it was, and the output matches the
    oracle's decode over the appended cache."""
    lens = [1, 15, 16, 17, 300, 2049, 64, 5, 1000, 33]
    Hkv = 2
    kc, vc, tables, q, kn, vn, pos, slots, cl = _step_case(lens, Hkv, G, d, 640 + d + G + P)
    ks, vs, theta, scale = 1 / 16, 1 / 12, 5e5, 1 / math.sqrt(d)
    qg, kvg = q.to(DEV), e4m3_pack(kc, vc).to(DEV)
    out = torch.full((len(lens), Hkv * G, d), float("nan"), device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.decode_step_e4m3(qg, kn.to(DEV), vn.to(DEV), pos.to(DEV), slots.to(DEV), kvg,
                         tables.to(DEV), cl.to(DEV), theta, scale, ks, vs, out,
                         partition_tokens=P, cluster=cluster, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    kco, vco, want = _oracle_step(kc, vc, tables, q, kn, vn, pos, slots, cl, theta, scale, ks, vs)
    kcg, vcg = (h.cpu() for h in e4m3_halves(kvg))
    assert torch.equal(kcg, kco), f"k codes differ at {(kcg != kco).nonzero()[:4].tolist()}"
    assert torch.equal(vcg, vco), f"v codes differ at {(vcg != vco).nonzero()[:4].tolist()}"
    assert torch.equal(qg.cpu(), q), "q must be read only"
    _check(out, want, f"e4m3 step d{d} G{G} P{P} cluster{cluster}")


def test_decode_step_e4m3_equals_two_calls_bytes():
    """The 64-sequence ragged batch (32/8 heads, d 64, U[128, 4096]): the
    fused step leaves the same cache bytes as kv_append_e4m3 and its output
    agrees with the two-call decode within rounding; both match the oracle."""
    g = _gen(650)
    B, Hkv, G, d = 64, 8, 4, 64
    lens = [L + 1 for L in torch.randint(128, 4097, (B,), generator=g).tolist()]
    kc, vc, tables, q, kn, vn, pos, slots, cl = _step_case(lens, Hkv, G, d, 651)
    ks, vs, theta, scale = 1 / 16, 1 / 16, 5e5, 0.125
    dev = [t.to(DEV) for t in (q, kn, vn, pos, slots, tables, cl)]
    qg, kng, vng, posg, slg, tg, clg = dev
    kv1, kv2 = e4m3_pack(kc, vc).to(DEV), e4m3_pack(kc, vc).to(DEV)
    out1 = torch.empty(B, Hkv * G, d, device=DEV)
    out2 = torch.empty(B, Hkv * G, d, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.decode_step_e4m3(qg, kng, vng, posg, slg, kv1, tg, clg, theta, scale, ks, vs, out1,
                         device_error=err)
    q2 = qg.clone()
    pkv.kv_append_e4m3(q2, kng, vng, posg, slg, kv2, theta, ks, vs, device_error=err)
    pkv.paged_attention_decode_e4m3(q2, kv2, tg, clg, scale, ks, vs, out2, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(kv1, kv2), "fused and two-call cache bytes differ"
    kco, vco, want = _oracle_step(kc, vc, tables, q, kn, vn, pos, slots, cl, theta, scale, ks, vs)
    assert torch.equal(kv1.cpu(), e4m3_pack(kco, vco)), "cache bytes differ from the oracle's"
    _check(out1, want, "fused ragged batch")
    _check(out2, want, "two-call ragged batch")


def test_decode_step_e4m3_edge_cases():
    """A padding slot (-1: not appended), a slot that is not the table's
    (flagged, not appended) and an empty context (zero output, token
    appended), against the oracle's append + decode of the same intent."""
    lens = [40, 40, 40, 0, 33]
    Hkv, G, d = 2, 4, 64
    kc, vc, tables, q, kn, vn, pos, slots, cl = _step_case(lens, Hkv, G, d, 660)
    slots_gpu = slots.clone()
    slots_gpu[0] = -1
    slots_gpu[1] = int(tables[1, 0]) * BS + 3
    slots_gpu[3] = int(tables[3, 0]) * BS + 9       # empty context: appended here
    slots_or = slots_gpu.clone()
    slots_or[1] = -1                               # the oracle sees "not appended"
    ks, vs, theta, scale = 1 / 16, 1 / 16, 1e4, 0.125
    kvg = e4m3_pack(kc, vc).to(DEV)
    out = torch.full((len(lens), Hkv * G, d), float("nan"), device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.decode_step_e4m3(q.to(DEV), kn.to(DEV), vn.to(DEV), pos.to(DEV), slots_gpu.to(DEV), kvg,
                         tables.to(DEV), cl.to(DEV), theta, scale, ks, vs, out,
                         device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pkv.DEVERR_SLOT
    kco, vco, want = _oracle_step(kc, vc, tables, q, kn, vn, pos, slots_or, cl, theta, scale,
                                  ks, vs)
    want[3].zero_()
    kcg, vcg = (h.cpu() for h in e4m3_halves(kvg))
    assert torch.equal(kcg, kco) and torch.equal(vcg, vco), "cache bytes"
    _check(out, want, "e4m3 step edge cases")


@pytest.mark.parametrize("window", [1, 16, 100, 5000])
def test_decode_step_e4m3_window(window):
    """The one-launch step with a sliding window: the same bytes as the
    append, the output of the windowed oracle decode; every byte no query
    may read is random (NaN codes included) in the pool."""
    lens = [1, 17, 300, 2049, 1000]
    Hkv, G, d = 2, 4, 128
    kc, vc, tables, q, kn, vn, pos, slots, cl = _step_case(lens, Hkv, G, d, 670 + window)
    ks, vs, theta, scale = 1 / 16, 1 / 16, 5e5, 1 / math.sqrt(d)
    kvg = e4m3_pack(kc, vc).to(DEV)
    out = torch.full((len(lens), Hkv * G, d), float("nan"), device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.decode_step_e4m3(q.to(DEV), kn.to(DEV), vn.to(DEV), pos.to(DEV), slots.to(DEV), kvg,
                         tables.to(DEV), cl.to(DEV), theta, scale, ks, vs, out,
                         partition_tokens=64, device_error=err, sliding_window=window)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    kco, vco, want = _oracle_step(kc, vc, tables, q, kn, vn, pos, slots, cl, theta, scale, ks, vs,
                                  window=window)
    kcg, vcg = (h.cpu() for h in e4m3_halves(kvg))
    assert torch.equal(kcg, kco) and torch.equal(vcg, vco), "cache bytes"
    _check(out, want, f"e4m3 step window {window}")
