"""Cascade decode (shared prefix blocks read once per group) vs the fp64
oracle's plain decode, through the C ABI (GPU only).

The cascade call must give the plain decode's result: the oracle decodes
every sequence over its own block table, with no knowledge of the groups.
The oracle's inputs are host copies taken before any GPU call, and the
oracle performs its own append (RoPE on q and k, the new rows written into
their slots): no value the CUDA path produced reaches it.
Bar: max-abs error <= 2e-3 (bf16 inputs, fp32 output).
"""
from __future__ import annotations

import pytest
import torch

import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200 import workloads as W
from tests.parity_util import TOL_BF16, SubProblem

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _grouped(lens, group, prefix_tokens, G, Hkv, d, seed):
    w = W.build_workload("cascade", lens, G * Hkv, Hkv, d, torch.bfloat16, 1e4, seed=seed,
                         device=DEV, pool_factor=1.2, prefix_group=group,
                         prefix_tokens=prefix_tokens)
    # the oracle's inputs, copied before the CUDA path touches anything
    sub = SubProblem(w, range(w.B))
    # rotate q and append the new token the usual way (two calls)
    pkv.kv_append(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache, w.v_cache,
                  w.rope_theta)
    B = w.B
    starts = list(range(0, B, group)) + [B]
    group_start = torch.tensor(starts, dtype=torch.int32, device=DEV)
    cached = w.cached_lens.to(torch.int64)
    shared = torch.minimum(cached // 16, torch.full_like(cached, prefix_tokens // 16)) * 16
    return w, sub, group_start, shared.to(torch.int32), group


def _oracle(sub):
    """The oracle's own append then plain decode, on the pristine copies."""
    return sub.oracle_step(nthreads=8)[3]


def _check(got, want, what):
    got = got.double().cpu()
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    err = (got - want).abs()
    assert err.max().item() <= TOL_BF16, f"{what}: max err {err.max().item():.3e}"


def _run(w, group_start, shared, max_group, P=0, err=None, window=0):
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
    pkv.paged_attention_decode_cascade(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                       group_start, shared, max_group, w.scale, out,
                                       partition_tokens=P, device_error=err,
                                       sliding_window=window)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("d,G,group,P", [(64, 4, 4, 0), (64, 4, 8, 128), (64, 8, 4, 64),
                                         (128, 4, 4, 256), (64, 1, 16, 0), (64, 4, 16, 512)])
def test_cascade_matches_plain_decode(d, G, group, P):
    lens = [1500, 300, 40, 255, 2000, 256, 16, 700, 1024, 77, 900, 260, 2047, 511, 5, 3000]
    w, sub, gs, shared, group = _grouped(lens, group, 512, G, 2, d, seed=400 + d + G + group)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = _run(w, gs, shared, group, P=P, err=err)
    assert int(err.item()) == 0
    _check(out, _oracle(sub), f"cascade d{d} G{G} group{group} P{P}")
    # and the same numbers as the plain decode call, up to rounding
    plain = torch.empty_like(out)
    pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                               w.scale, plain, partition_tokens=P)
    torch.cuda.synchronize()
    assert (out - plain).abs().max().item() < 1e-4


@pytest.mark.parametrize("window,P", [(1, 0), (16, 64), (100, 0), (300, 128), (600, 0),
                                      (1100, 256), (5000, 0)])
def test_cascade_with_window_matches_windowed_decode(window, P):
    """Each query attends to its last `window` tokens: windows that start past
    the shared prefix (empty shared slot), inside it, and before it, against
    the oracle's windowed decode of every sequence over its own table.  The
    tokens the kernels may skip are NaN in the cache, so a stray read shows
    up."""
    lens = [1500, 300, 40, 255, 2000, 256, 16, 700, 1024, 77, 900, 260, 2047, 511, 5, 3000]
    w, sub, gs, shared, group = _grouped(lens, 4, 512, 4, 2, 64, seed=470 + window)
    # NaN (in the GPU's cache only) in the tokens no query reads: those of a
    # sequence's own pages before its window, and those of the group's shared
    # pages before the first token any member attends.  (Shared tokens from
    # there on are the group's prompt prefix, finite cache contents, which a
    # member may skip under its own window while another reads them.)
    L = w.decode_lens.to(torch.int64).cpu()
    lo = torch.clamp(L - window, min=0)
    sh = shared.to(torch.int64).cpu()
    tables = w.block_tables.to(torch.int64).cpu()
    nan_k, nan_v = w.k_cache.clone(), w.v_cache.clone()
    for b in range(w.B):
        g0 = (b // group) * group
        members = range(g0, min(g0 + group, w.B))
        with_keys = [int(lo[m]) for m in members if lo[m] < sh[m]]
        first_read = min(with_keys) if with_keys else int(max(sh[m] for m in members))
        t = torch.arange(int(lo[b]))
        t = t[(t >= sh[b]) | (t < first_read)]
        if t.numel() == 0:
            continue
        blk, row = tables[b, t // 16].to(DEV), (t % 16).to(DEV)
        nan_k[blk, :, row] = float("nan")
        nan_v[blk, :, row] = float("nan")
    w.k_cache.copy_(nan_k)
    w.v_cache.copy_(nan_v)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = _run(w, gs, shared, group, P=P, err=err, window=window)
    assert int(err.item()) == 0
    _check(out, sub.oracle_step(nthreads=8, window=window)[3],
           f"cascade window {window} P{P}")


def test_cascade_edge_cases():
    """A whole context inside the shared prefix, a sequence in no group, a
    group of one, a sequence with no shared tokens in a group, an empty
    context (all-zero row), and a member whose shared block id differs from
    its group's (flagged)."""
    lens = [512, 700, 512, 100, 900, 30, 640, 640]
    w, sub, gs, shared, _ = _grouped(lens, 4, 512, 4, 2, 64, seed=431)
    # the first sequence's decode length is 513 after the append: make its
    # context exactly the shared part (the oracle's copy likewise)
    w.decode_lens[0] = 512
    sub.decode_lens[0] = 512
    # group layout: [0, 4) and [4, 6); sequences 6 and 7 in no group
    gs = torch.tensor([0, 4, 5, 6], dtype=torch.int32, device=DEV)   # group of one: [4, 5)
    shared[6:] = 0
    shared[5] = 0                       # in a group, nothing shared
    w.decode_lens[7] = 0                # empty context
    sub.decode_lens[7] = 0
    out = _run(w, gs, shared, 4)
    want = _oracle(sub)
    assert not want[7].any()            # the oracle's empty context is a zero row too
    _check(out, want, "cascade edge cases")
    assert not out[7].any()
    # a member whose shared block differs from the group's: flagged
    w.block_tables[2, 3] = w.block_tables[6, 20]
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    _run(w, gs, shared, 4, err=err)
    assert int(err.item()) & pkv.DEVERR_PREFIX


def test_cascade_workspace_counters_return_to_zero():
    w, sub, gs, shared, group = _grouped([800, 600, 1200, 300] * 2, 4, 256, 4, 8, 64, seed=433)
    need = pkv.decode_cascade_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks)
    ws = pkv.new_workspace(need, DEV)
    outs = []
    for _ in range(2):
        out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
        pkv.paged_attention_decode_cascade(w.q, w.k_cache, w.v_cache, w.block_tables,
                                           w.decode_lens, gs, shared, group, w.scale, out,
                                           workspace=ws)
        torch.cuda.synchronize()
        assert not ws[:pkv.SCHED_BYTES].any()
        outs.append(out)
    assert torch.equal(outs[0], outs[1])
    _check(outs[0], _oracle(sub), "cascade, reused workspace")
