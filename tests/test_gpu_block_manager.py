"""The host block manager feeding the device calls (GPU only).

Sequences are admitted through ``BlockManager``; their prompt K/V are
written by ``kv_append`` only into the slots the manager hands out (reused
prefix blocks are skipped), one decode token is appended per sequence, and
the plain and cascade decodes run over the manager's block tables.

The K/V of a token is a seeded function of the token ids up to and
including it, as in a model, so a reused block holds exactly what the
sequence would have written itself.  The oracle recomputes every sequence
from scratch in a private, unshared cache (its own RoPE and append), so the
check covers the reuse decisions as well as the kernels.
Bar: max-abs error <= 2e-3 (bf16 inputs, fp32 output).
"""
from __future__ import annotations

import random

import pytest
import torch

import oracle
import paged_kv_cache_484_b200 as pkv
from tests.parity_util import TOL_BF16

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
BS = 16
HKV, G, D = 2, 4, 64
HQ = HKV * G
THETA = 1e4


def _prefix_seed(tokens, p):
    h = 1469598103934665603
    for t in tokens[: p + 1]:
        h = ((h ^ (t + 1)) * 1099511628211) & 0xFFFFFFFFFFFF
    return h


def _token_kv(tokens, p):
    g = torch.Generator().manual_seed(_prefix_seed(tokens, p))
    kv = torch.randn(2, HKV, D, generator=g)
    return kv[0].to(torch.bfloat16), kv[1].to(torch.bfloat16)


def _write_tokens(entries, k_cache, v_cache):
    """entries: list of (tokens, position, slot); one kv_append call."""
    T = len(entries)
    k = torch.stack([_token_kv(t, p)[0] for t, p, _ in entries])
    v = torch.stack([_token_kv(t, p)[1] for t, p, _ in entries])
    pos = torch.tensor([p for _, p, _ in entries], dtype=torch.int64)
    slots = torch.tensor([s for _, _, s in entries], dtype=torch.int64)
    q = torch.zeros(T, HQ, D, dtype=torch.bfloat16, device=DEV)
    pkv.kv_append(q, k.to(DEV), v.to(DEV), pos.to(DEV), slots.to(DEV), k_cache, v_cache, THETA)


def _oracle_fresh(seqs, q):
    """Every sequence recomputed into its own blocks by the oracle."""
    B = len(seqs)
    MB = max((len(t) + BS - 1) // BS for t in seqs)
    kc = torch.zeros(B * MB, HKV, BS, D, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    tables = torch.arange(B * MB, dtype=torch.int32).view(B, MB)
    qq = q.clone()
    for b, toks in enumerate(seqs):
        n = len(toks)
        k = torch.stack([_token_kv(toks, p)[0] for p in range(n)])
        v = torch.stack([_token_kv(toks, p)[1] for p in range(n)])
        pos = torch.arange(n, dtype=torch.int64)
        slots = b * MB * BS + pos
        qb = torch.zeros(n, HQ, D, dtype=torch.bfloat16)
        qb[n - 1] = qq[b]
        oracle.kv_append(qb, k, v, pos, slots, kc, vc, THETA)
        qq[b] = qb[n - 1]
    lens = torch.tensor([len(t) for t in seqs], dtype=torch.int32)
    return oracle.paged_attention_decode(qq, kc, vc, tables, lens, D ** -0.5, nthreads=8)


def _admit(bm, sid, prompt, k_cache, v_cache):
    shared = bm.add_sequence(sid, prompt)
    slots = bm.prompt_slots(sid, len(prompt))
    assert (slots[:shared] == -1).all() and (slots[shared:] >= 0).all()
    entries = [(prompt, p, int(slots[p])) for p in range(shared, len(prompt))]
    if entries:
        _write_tokens(entries, k_cache, v_cache)
    return shared


def _rotate_q(q, seqs, k_cache, v_cache):
    """The step's RoPE of q on the device: a kv_append whose slots are all
    -1 rotates q and writes nothing."""
    n = len(seqs)
    q_dev = q.to(DEV)
    zeros = torch.zeros(n, HKV, D, dtype=torch.bfloat16, device=DEV)
    pos = torch.tensor([len(t) - 1 for t in seqs], dtype=torch.int64, device=DEV)
    pkv.kv_append(q_dev, zeros, zeros, pos, torch.full((n,), -1, dtype=torch.int64, device=DEV),
                  k_cache, v_cache, THETA)
    return q_dev


def _decode_and_check(bm, ids, seqs, k_cache, v_cache, q, MB, groups):
    q_rot_dev = _rotate_q(q, seqs, k_cache, v_cache)
    tables = torch.stack([bm.block_table(s, MB)[0] for s in ids]).to(DEV)
    lens = torch.tensor([bm.block_table(s, MB)[1] for s in ids], dtype=torch.int32, device=DEV)
    want = _oracle_fresh(seqs, q)
    out = torch.empty(len(ids), HQ, D, dtype=torch.float32, device=DEV)
    pkv.paged_attention_decode(q_rot_dev, k_cache, v_cache, tables, lens, D ** -0.5, out)
    torch.cuda.synchronize()
    assert (out.double().cpu() - want).abs().max().item() <= TOL_BF16
    # cascade over consecutive groups; shared tokens = the leading blocks
    # every member has in common with the group's first member
    host_tables = tables.cpu()
    shared = torch.zeros(len(ids), dtype=torch.int32)
    starts = [0]
    for gs, ge in groups:
        for b in range(gs + 1, ge):
            n = 0
            while (n < MB and host_tables[b, n] >= 0 and host_tables[b, n] == host_tables[gs, n]
                   and (n + 1) * BS <= int(lens[b]) - 1):
                n += 1
            shared[b] = n * BS
        shared[gs] = int(shared[gs + 1: ge].max()) if ge - gs > 1 else 0
        starts.append(ge)
    casc = torch.empty_like(out)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.paged_attention_decode_cascade(q_rot_dev, k_cache, v_cache, tables, lens,
                                       torch.tensor(starts, dtype=torch.int32, device=DEV),
                                       shared.to(DEV), max(ge - gs for gs, ge in groups),
                                       D ** -0.5, casc, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert (casc.double().cpu() - want).abs().max().item() <= TOL_BF16
    return shared


def test_block_manager_prefix_reuse_end_to_end():
    rng = random.Random(11)
    NB, MB = 96, 12
    k_cache = torch.zeros(NB, HKV, BS, D, dtype=torch.bfloat16, device=DEV)
    v_cache = torch.zeros_like(k_cache)
    bm = pkv.BlockManager(NB, BS)
    sys_a = [rng.randrange(1000) for _ in range(70)]
    sys_b = [rng.randrange(1000) for _ in range(40)]
    prompts = [sys_a + [rng.randrange(1000) for _ in range(rng.randrange(3, 60))] for _ in range(4)]
    prompts += [sys_b + [rng.randrange(1000) for _ in range(rng.randrange(3, 60))] for _ in range(4)]
    ids = list(range(8))
    shared = [_admit(bm, s, p, k_cache, v_cache) for s, p in zip(ids, prompts)]
    assert shared == [0, 64, 64, 64, 0, 32, 32, 32]

    # one decode token per sequence: appended through the manager's slots
    seqs = [p + [rng.randrange(1000)] for p in prompts]
    slots = [bm.append(s, t[-1]) for s, t in zip(ids, seqs)]
    gen = torch.Generator().manual_seed(5)
    q = torch.randn(len(ids), HQ, D, generator=gen).to(torch.bfloat16)
    _write_tokens([(t, len(t) - 1, s) for t, s in zip(seqs, slots)], k_cache, v_cache)
    casc_shared = _decode_and_check(bm, ids, seqs, k_cache, v_cache, q, MB, [(0, 4), (4, 8)])
    assert casc_shared.tolist() == [64, 64, 64, 64, 32, 32, 32, 32]

    # the group's first owner leaves; its prefix blocks stay cached and a
    # newcomer with the same system prompt reuses them
    bm.free_sequence(0)
    newcomer = sys_a + [rng.randrange(1000) for _ in range(9)]
    assert _admit(bm, 100, newcomer, k_cache, v_cache) == 64
    seq_new = newcomer + [rng.randrange(1000)]
    slot = bm.append(100, seq_new[-1])
    _write_tokens([(seq_new, len(seq_new) - 1, slot)], k_cache, v_cache)
    ids2 = [100, 1, 2, 3]
    seqs2 = [seq_new] + seqs[1:4]
    q2 = torch.randn(4, HQ, D, generator=gen).to(torch.bfloat16)
    _decode_and_check(bm, ids2, seqs2, k_cache, v_cache, q2, MB, [(0, 4)])
