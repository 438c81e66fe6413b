"""Sliding-window decode through the C ABI vs the fp64 oracle (GPU only).

Each query attends to the last W tokens of its context.  The cases cover a
window that starts inside a page, on a page boundary, inside the first
partition and beyond the context (no effect), W = 1, every partitioning
mode (one partition, split with the combine kernel, cluster merge), the
tensor-core and CUDA-core kernels, bf16 / fp32 caches and the 8-bit cache.
Pages before the window hold NaN, so a page or token read outside the
window shows up as a non-finite or wrong output.
Bars: 1e-5 (fp32 inputs), 2e-3 (bf16 inputs), fp32 output.
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
import paged_kv_cache_484_b200 as pkv
from tests.parity_util import TOL_BF16, TOL_F32

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
BS = 16
LENS = [1, 15, 16, 17, 300, 2049, 64, 0, 5, 1000]


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def _paged(lens, Hkv, d, dtype, seed, window):
    """Random pool and tables; every token before a sequence's window is NaN
    (it must not be read), the rest N(0, 1)."""
    g = _gen(seed)
    need = [max(1, math.ceil(L / BS)) for L in lens]
    NB = sum(need) + 3
    perm = torch.randperm(NB, generator=g)
    tables = torch.full((len(lens), max(need)), -1, dtype=torch.int32)
    kc = torch.randn(NB, Hkv, BS, d, generator=g).to(dtype)
    vc = torch.randn(NB, Hkv, BS, d, generator=g).to(dtype)
    c = 0
    for b, L in enumerate(lens):
        ids = perm[c:c + need[b]]
        c += need[b]
        tables[b, :need[b]] = ids.to(torch.int32)
        t = torch.arange(max(0, L - window) if window else 0)
        kc[ids[t // BS], :, t % BS] = float("nan")
        vc[ids[t // BS], :, t % BS] = float("nan")
    return kc, vc, tables


def _oracle_input(x):
    """The oracle reads only tokens inside the window; give it zeros where the
    GPU input holds NaN so that a wrong oracle read would not hide."""
    return torch.nan_to_num(x, nan=0.0)


@pytest.mark.parametrize("dtype,d,G,simt", [
    (torch.bfloat16, 64, 4, False), (torch.bfloat16, 64, 8, False), (torch.bfloat16, 128, 4, False),
    (torch.bfloat16, 64, 1, False), (torch.bfloat16, 64, 4, True), (torch.float32, 64, 4, False),
    (torch.float32, 128, 2, False),
])
@pytest.mark.parametrize("W,P,cluster", [
    (1, 0, True), (15, 0, True), (16, 64, False), (17, 16, False), (100, 0, True),
    (100, 48, True), (1000, 128, False), (5000, 0, True),
])
def test_window_matches_oracle(dtype, d, G, simt, W, P, cluster):
    Hkv = 2
    kc, vc, tables = _paged(LENS, Hkv, d, dtype, seed=700 + d + G + W, window=W)
    q = torch.randn(len(LENS), Hkv * G, d, generator=_gen(701 + W)).to(dtype)
    cl = torch.tensor(LENS, dtype=torch.int32)
    out = torch.empty(len(LENS), Hkv * G, d, dtype=torch.float32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.paged_attention_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), tables.to(DEV), cl.to(DEV),
                               d ** -0.5, out, partition_tokens=P, force_simt=simt,
                               cluster=cluster, device_error=err, sliding_window=W)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle.paged_attention_decode(q, _oracle_input(kc), _oracle_input(vc), tables, cl,
                                         d ** -0.5, nthreads=8, window=W)
    got = out.double().cpu()
    assert torch.isfinite(got).all(), "a token outside the window was read"
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert (got - want).abs().max().item() <= tol


@pytest.mark.parametrize("d,W,P", [(64, 33, 0), (64, 1000, 64), (128, 17, 0), (64, 1, 16)])
def test_window_e4m3_matches_oracle(d, W, P):
    Hkv, G = 2, 4
    g = _gen(710 + d + W)
    need = [max(1, math.ceil(L / BS)) for L in LENS]
    NB = sum(need) + 3
    perm = torch.randperm(NB, generator=g)
    tables = torch.full((len(LENS), max(need)), -1, dtype=torch.int32)
    kc = (torch.randn(NB, Hkv, BS, d, generator=g) * 16).to(torch.float8_e4m3fn).view(torch.uint8)
    vc = (torch.randn(NB, Hkv, d, BS, generator=g) * 16).to(torch.float8_e4m3fn).view(torch.uint8)
    kc_gpu, vc_gpu = kc.clone(), vc.clone()
    c = 0
    for b, L in enumerate(LENS):
        ids = perm[c:c + need[b]]
        c += need[b]
        tables[b, :need[b]] = ids.to(torch.int32)
        t = torch.arange(max(0, L - W))        # NaN codes before the window
        kc_gpu[ids[t // BS], :, t % BS] = 0x7F
        vc_gpu[ids[t // BS], :, :, t % BS] = 0x7F
    q = torch.randn(len(LENS), Hkv * G, d, generator=g).to(torch.bfloat16)
    cl = torch.tensor(LENS, dtype=torch.int32)
    out = torch.empty(len(LENS), Hkv * G, d, dtype=torch.float32, device=DEV)
    from paged_kv_cache_484_b200.workloads import e4m3_pack
    pkv.paged_attention_decode_e4m3(q.to(DEV), e4m3_pack(kc_gpu, vc_gpu).to(DEV), tables.to(DEV),
                                    cl.to(DEV), d ** -0.5, 1 / 16, 1 / 16, out,
                                    partition_tokens=P, sliding_window=W)
    torch.cuda.synchronize()
    want = oracle.paged_attention_decode_e4m3(q, kc, vc, tables, cl, d ** -0.5, 1 / 16, 1 / 16,
                                              nthreads=8, window=W)
    got = out.double().cpu()
    assert torch.isfinite(got).all(), "a token outside the window was read"
    assert (got - want).abs().max().item() <= TOL_BF16


def test_window_on_the_ragged_batch():
    """64 sequences of U[128, 4096] tokens, 32/8 heads, window 1024, at the
    partition length the library picks: against the oracle."""
    g = _gen(720)
    lens = torch.randint(128, 4097, (64,), generator=g).tolist()
    kc, vc, tables = _paged(lens, 8, 64, torch.bfloat16, seed=721, window=1024)
    q = torch.randn(64, 32, 64, generator=g).to(torch.bfloat16)
    cl = torch.tensor(lens, dtype=torch.int32)
    out = torch.empty(64, 32, 64, dtype=torch.float32, device=DEV)
    pkv.paged_attention_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), tables.to(DEV), cl.to(DEV),
                               0.125, out, sliding_window=1024)
    torch.cuda.synchronize()
    want = oracle.paged_attention_decode(q, _oracle_input(kc), _oracle_input(vc), tables, cl,
                                         0.125, nthreads=16, window=1024)
    got = out.double().cpu()
    assert torch.isfinite(got).all()
    assert (got - want).abs().max().item() <= TOL_BF16


@pytest.mark.parametrize("d,G", [(64, 4), (128, 4), (64, 8)])
@pytest.mark.parametrize("W,P,cluster", [
    (1, 0, True), (16, 64, False), (17, 0, True), (100, 48, True), (1000, 128, False),
    (5000, 0, True),
])
def test_fused_step_with_window_matches_oracle(d, G, W, P, cluster):
    """pkv_decode_step_window: the new token appended inside the decode kernel,
    each query attending to its last W tokens (the new one included).  The
    oracle appends with its own RoPE, then decodes with the window, on host
    copies taken before the GPU step; every cached token before a window is
    NaN on the GPU."""
    from paged_kv_cache_484_b200 import workloads as W_
    from tests.parity_util import SubProblem, check_within_one_bf16_ulp
    lens = [300, 0, 15, 16, 2048, 777, 64, 5]
    w = W_.build_workload("window-step", lens, G * 2, 2, d, torch.bfloat16, 5e5,
                          seed=760 + d + G + W, device=DEV, pool_factor=1.2)
    sub = SubProblem(w, range(w.B))
    # tokens before every window hold NaN in the GPU cache (never read)
    tables = w.block_tables.cpu()
    blks, rows = [], []
    for b, L in enumerate(w.decode_lens.tolist()):
        t = torch.arange(max(0, L - W))
        blks.append(tables[b, t // BS].long())
        rows.append(t % BS)
    blks, rows = torch.cat(blks).to(DEV), torch.cat(rows).to(DEV)
    w.k_cache[blks, :, rows] = float("nan")
    w.v_cache[blks, :, rows] = float("nan")
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
    pkv.decode_step(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache, w.v_cache,
                    w.block_tables, w.decode_lens, w.rope_theta, w.scale, out,
                    partition_tokens=P, device_error=err, cluster=cluster, sliding_window=W)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    q, kc, vc = sub.q.clone(), sub.k_cache.clone(), sub.v_cache.clone()
    oracle.kv_append(q, sub.k_new.clone(), sub.v_new.clone(), sub.positions, sub.slots, kc, vc,
                     sub.theta)
    want = oracle.paged_attention_decode(q, kc, vc, sub.tables, sub.decode_lens, sub.scale,
                                         nthreads=8, window=W)
    got = out.double().cpu()
    assert torch.isfinite(got).all()
    assert (got - want).abs().max().item() <= TOL_BF16
    # the appended rows: within one bf16 ulp of the oracle's
    slots = w.slot_mapping.cpu()
    for b in range(w.B):
        s_g, s_o = int(slots[b]), int(sub.slots[b])
        check_within_one_bf16_ulp(w.k_cache[s_g // BS, :, s_g % BS].cpu(), kc[s_o // BS, :, s_o % BS],
                                  f"appended k of sequence {b}")
        assert torch.equal(w.v_cache[s_g // BS, :, s_g % BS].cpu(), vc[s_o // BS, :, s_o % BS])
