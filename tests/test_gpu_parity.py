"""CUDA path vs the fp64 oracle, through the C ABI (GPU only).

Bars: cache placement and v bit-exact; appended k and rotated q within one
bf16 ulp of the oracle; attention output max-abs error <= 1e-5 for fp32
inputs and <= 2e-3 for bf16 inputs (fp32 output), plus half a bf16 ulp when
the output itself is bf16.
"""
from __future__ import annotations

import pytest
import torch

import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200 import workloads as W
from tests.parity_util import (SubProblem, check_decode, check_decode_bf16_out,
                               check_within_one_bf16_ulp, gpu_step, sample_pairs)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _placement_and_append(w, before_k, before_v, sub, q_gpu, q_or, kc_or, vc_or, q_in=None):
    """Exactly the slot rows changed; v bit copy; k within one bf16 ulp; q
    rotated in place within one bf16 ulp (two calls) or untouched (one-launch
    step, ``q_in`` given)."""
    bs = w.block_size
    itype = torch.int16 if w.dtype == torch.bfloat16 else torch.int32
    changed = (w.k_cache.view(itype) != before_k.view(itype)).any(-1) | \
              (w.v_cache.view(itype) != before_v.view(itype)).any(-1)      # [NB, Hkv, bs]
    want = torch.zeros_like(changed)
    slots = w.slot_mapping.long()
    want[slots // bs, :, slots % bs] = True
    # a row may be rewritten with identical bits by chance only for k; v rows
    # of a fresh N(0,1) draw differ from the old contents with certainty
    extra = changed & ~want
    assert not extra.any(), f"rows outside the slots changed: {extra.nonzero()[:4].tolist()}"
    vrows_changed = (w.v_cache.view(itype) != before_v.view(itype)).any(-1)
    assert torch.equal(vrows_changed, want), "v rows written != slots"
    # values of the sampled sequences
    for i, b in enumerate(sub.seqs):
        s = int(w.slot_mapping[b])
        so = int(sub.slots[i])
        gk = w.k_cache[s // bs, :, s % bs].cpu()
        gv = w.v_cache[s // bs, :, s % bs].cpu()
        ok_ = kc_or[so // bs, :, so % bs]
        ov = vc_or[so // bs, :, so % bs]
        assert torch.equal(gv.view(itype), ov.view(itype)), f"v bits, seq {b}"
        check_within_one_bf16_ulp(gk, ok_, f"appended k, seq {b}")
        if q_in is None:
            check_within_one_bf16_ulp(q_gpu[b].cpu(), q_or[i], f"rotated q, seq {b}")
    if q_in is not None:
        assert torch.equal(q_gpu, q_in), "decode_step must leave q untouched"


def _seq_sample(cfg, w):
    if cfg in (1, 2, 3):
        return list(range(w.B))
    lens = w.cached_lens.cpu()
    order = torch.argsort(lens)
    pick = set(order[:6].tolist()) | set(order[-6:].tolist()) | set(range(8, 16))
    pick |= set(torch.randperm(w.B, generator=torch.Generator().manual_seed(5))[:6].tolist())
    if cfg == 5:
        pick = {0, 7, 15}
    return sorted(pick)


@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "one_launch"])
@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_named_workload_step(cfg, fused):
    """One full step (append + decode) of each named workload, at full size,
    in the launch configuration the benchmark times: as the two calls, and as
    the single-launch decode_step."""
    w = W.make_config(cfg, device=DEV)
    seqs = _seq_sample(cfg, w)
    sub = SubProblem(w, seqs)
    full_heads = cfg in (1, 2, 3)
    pairs = None if full_heads else sample_pairs(w, seqs, n_heads_per_seq=4, seed=cfg)
    before_k = w.k_cache.clone()
    before_v = w.v_cache.clone()
    q_in = w.q.clone()

    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    out32 = gpu_step(w, out_dtype=torch.float32, fused=fused, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    q_or, kc_or, vc_or, ref = sub.oracle_step(nthreads=16, pairs=pairs)
    _placement_and_append(w, before_k, before_v, sub, w.q, q_or, kc_or, vc_or,
                          q_in=q_in if fused else None)
    del before_k, before_v

    sel = torch.tensor(seqs)
    got = out32.cpu()[sel]
    if pairs is None:
        check_decode(got, ref, w.dtype, f"cfg{cfg} f32 out")
    else:
        g = torch.stack([got[i, h] for i, h in pairs.tolist()])
        r = torch.stack([ref[i, h] for i, h in pairs.tolist()])
        check_decode(g, r, w.dtype, f"cfg{cfg} f32 out (sampled)")

    if w.dtype == torch.bfloat16:
        # the benchmark's output dtype, on the same state: the two-call path
        # decodes again with the rotated q; the one-launch step runs again (it
        # rewrites the same new rows and leaves q as it was)
        out16 = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=DEV)
        if fused:
            pkv.decode_step(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache,
                            w.v_cache, w.block_tables, w.decode_lens, w.rope_theta, w.scale,
                            out16)
        else:
            pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                       w.scale, out16)
        got16 = out16.cpu()[sel]
        if pairs is None:
            check_decode_bf16_out(got16, ref, f"cfg{cfg} bf16 out")
        else:
            g = torch.stack([got16[i, h] for i, h in pairs.tolist()])
            r = torch.stack([ref[i, h] for i, h in pairs.tolist()])
            check_decode_bf16_out(g, r, f"cfg{cfg} bf16 out (sampled)")
    del q_in


LENS = [1, 15, 16, 17, 63, 64, 65, 127, 129, 300, 1000, 2049]


@pytest.mark.parametrize("dtype,d,G,simt", [
    (torch.float32, 64, 1, True), (torch.float32, 64, 4, True), (torch.float32, 128, 8, True),
    (torch.float32, 128, 2, True),
    (torch.bfloat16, 64, 1, False), (torch.bfloat16, 64, 2, False), (torch.bfloat16, 64, 4, False),
    (torch.bfloat16, 64, 8, False), (torch.bfloat16, 128, 1, False), (torch.bfloat16, 128, 2, False),
    (torch.bfloat16, 128, 4, False), (torch.bfloat16, 128, 8, False),
    (torch.bfloat16, 64, 4, True), (torch.bfloat16, 128, 8, True), (torch.bfloat16, 64, 1, True),
])
@pytest.mark.parametrize("P", [0, 16, 64, 512])
@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "one_launch"])
def test_shapes_and_partitions(dtype, d, G, simt, P, fused):
    Hkv = 2
    lens = [L - 1 for L in LENS]
    w = W.build_workload("shapes", lens, G * Hkv, Hkv, d, dtype, 1e4, seed=100 + d + G, device=DEV,
                         pool_factor=1.3)
    if not fused:
        # one empty context: its output must be zeros (the fused step's
        # precondition excludes it; tested separately)
        w.decode_lens[5] = 0
    sub = SubProblem(w, range(w.B))
    q_in = w.q.clone()
    out = gpu_step(w, out_dtype=torch.float32, partition_tokens=P, force_simt=simt, fused=fused)
    torch.cuda.synchronize()
    q_or, kc_or, _, ref = sub.oracle_step()
    if not fused:
        ref[5].zero_()
    check_decode(out, ref, dtype, f"{dtype} d{d} G{G} simt={simt} P={P} fused={fused}")
    if not fused:
        assert torch.equal(out[5].cpu(), torch.zeros_like(out[5].cpu()))
        check_within_one_bf16_ulp(w.q.cpu(), q_or, "rotated q")
    else:
        assert torch.equal(w.q, q_in)


def test_partition_length_does_not_change_result():
    w = W.build_workload("plen", [3000, 700, 5], 32, 8, 64, torch.bfloat16, 5e5, seed=7, device=DEV)
    pkv.kv_append(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache, w.v_cache,
                  w.rope_theta)
    outs = []
    for P in (16, 64, 256, 1024, 4096, 8192):
        o = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
        pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                   w.scale, o, partition_tokens=P)
        outs.append(o.cpu())
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() < 1e-4


def test_degenerate_contexts():
    """Length-1 context returns V exactly; identical keys and zero scale give
    the mean of V (the oracle computes the same definitions)."""
    d, Hkv, G = 64, 2, 4
    w = W.build_workload("degen", [0, 40, 40], G * Hkv, Hkv, d, torch.bfloat16, 1e4, seed=9,
                         device=DEV)
    bs = 16
    # sequence 1: all cached keys equal (and the appended one too, after RoPE: no,
    # so compare with the oracle which sees the same inputs)
    t1 = w.block_tables[1]
    for t in range(40):
        w.k_cache[t1[t // bs], :, t % bs] = w.k_cache[t1[0], :, 0]
    sub = SubProblem(w, range(w.B))
    out = gpu_step(w, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _, _, vc_or, ref = sub.oracle_step()
    check_decode(out, ref, torch.bfloat16, "degenerate")
    # length 1: exactly the appended v (fp32 output of a bf16 value)
    s = int(w.slot_mapping[0])
    v = w.v_cache[s // bs, :, s % bs].float()                       # [Hkv, d]
    assert torch.allclose(out[0], v.repeat_interleave(G, 0), rtol=1e-6, atol=0)
    # zero scale: mean of V over the context
    o0 = torch.empty_like(out)
    pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens, 0.0, o0)
    rows = [w.v_cache[w.block_tables[2][t // bs], :, t % bs].double() for t in range(41)]
    mean = torch.stack(rows).mean(0).repeat_interleave(G, 0)
    assert (o0[2].double() - mean).abs().max().item() < 2e-3


def test_many_sequences_at_the_limit():
    lens = (torch.arange(4096) % 37).tolist()
    w = W.build_workload("many", lens, 8, 8, 64, torch.bfloat16, 1e4, seed=11, device=DEV)
    seqs = [0, 1, 36, 37, 1000, 4095]
    sub = SubProblem(w, seqs)
    out = gpu_step(w, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _, _, _, ref = sub.oracle_step()
    check_decode(out.cpu()[torch.tensor(seqs)], ref, torch.bfloat16, "4096 sequences")


def test_empty_batch_is_a_no_op():
    q = torch.empty((0, 8, 64), dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((0, 8, 64), dtype=torch.bfloat16, device=DEV)
    pkv.paged_attention_decode(q, kc, kc, torch.zeros((0, 1), dtype=torch.int32, device=DEV),
                               torch.zeros((0,), dtype=torch.int32, device=DEV), 0.1, out)
    pkv.kv_append(q, torch.empty((0, 2, 64), dtype=torch.bfloat16, device=DEV),
                  torch.empty((0, 2, 64), dtype=torch.bfloat16, device=DEV),
                  torch.empty((0,), dtype=torch.int64, device=DEV),
                  torch.empty((0,), dtype=torch.int64, device=DEV), kc, kc, 1e4)
    torch.cuda.synchronize()


def test_fused_step_edge_cases():
    """decode_step with a padding slot (-1), a slot that is not the last
    token's table slot, and an empty context, against the oracle's append +
    decode of the same intent."""
    d, Hkv, G = 64, 2, 4
    w = W.build_workload("edges", [40, 40, 40, 0, 33], G * Hkv, Hkv, d, torch.bfloat16, 5e5, seed=21,
                         device=DEV, pool_factor=1.5)
    bs = 16
    # sequence 0: padding slot -> not appended, cached context attended as is
    w.slot_mapping[0] = -1
    # sequence 1: a slot that is not its last token's slot -> flagged, not appended
    good1 = int(w.slot_mapping[1])
    w.slot_mapping[1] = int(w.block_tables[1][0]) * bs + 3
    # sequence 3: context length 0 -> zero output, token appended as kv_append would
    w.decode_lens[3] = 0
    sub = SubProblem(w, range(w.B))
    sub.slots[0] = -1          # the oracle sees "not appended" for sequences 0 and 1 too
    sub.slots[1] = -1
    k_before = w.k_cache.clone()
    q_in = w.q.clone()
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = gpu_step(w, out_dtype=torch.float32, fused=True, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv.DEVERR_SLOT
    q_or, kc_or, vc_or, ref = sub.oracle_step()
    ref[3].zero_()
    check_decode(out, ref, torch.bfloat16, "fused edge cases")
    assert torch.equal(w.q, q_in)
    # sequence 1's intended slot and the bogus one were left untouched
    for s_ in (good1, int(w.block_tables[1][0]) * bs + 3):
        assert torch.equal(w.k_cache[s_ // bs, :, s_ % bs], k_before[s_ // bs, :, s_ % bs])
    # sequence 3 (empty context) was appended
    s3 = int(w.slot_mapping[3])
    so3 = int(sub.slots[3])
    check_within_one_bf16_ulp(w.k_cache[s3 // bs, :, s3 % bs].cpu(), kc_or[so3 // bs, :, so3 % bs],
                              "appended k of the empty context")


@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "one_launch"])
def test_claimed_work_items_repeat_exactly(fused):
    """CTAs claim work items from the workspace's counters: three calls that
    share one workspace give bit-identical outputs (an item's arithmetic does
    not depend on which CTA runs it), match the oracle, and leave the
    counters at zero after every call."""
    lens = [4000, 130, 2500, 17, 3333, 900, 64, 1, 4095, 2048] * 6
    w = W.build_workload("claims", lens, 32, 8, 64, torch.bfloat16, 5e5, seed=53, device=DEV)
    seqs = [0, 3, 7, 8, 59]
    sub = SubProblem(w, seqs)
    _, _, _, ref = sub.oracle_step()
    P = 128
    need = pkv.decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks, partition_tokens=P)
    ws = pkv.new_workspace(need, DEV)
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    outs = []
    for _ in range(3):
        w.k_cache.copy_(k0)
        w.v_cache.copy_(v0)
        q = w.q.clone()
        out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
        if fused:
            pkv.decode_step(q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache,
                            w.v_cache, w.block_tables, w.decode_lens, w.rope_theta, w.scale, out,
                            workspace=ws, partition_tokens=P)
        else:
            pkv.kv_append(q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache,
                          w.v_cache, w.rope_theta)
            pkv.paged_attention_decode(q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                       w.scale, out, workspace=ws, partition_tokens=P)
        torch.cuda.synchronize()
        assert not ws[:pkv.SCHED_BYTES].any(), "scheduler counters not back at zero"
        outs.append(out)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    check_decode(outs[0].cpu()[torch.tensor(seqs)], ref, torch.bfloat16, "claimed items")


@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "one_launch"])
def test_static_schedule_without_workspace(fused):
    """No workspace (allowed when no context is split): items are dealt out
    round-robin; same results as the oracle."""
    lens = [700, 1, 0, 512, 33, 1000, 999, 16]
    w = W.build_workload("static", lens, 16, 4, 128, torch.bfloat16, 1e4, seed=59, device=DEV)
    sub = SubProblem(w, list(range(w.B)))
    q_or, _, _, ref = sub.oracle_step()
    P = 1024
    assert pkv.decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks,
                                     partition_tokens=P) == pkv.SCHED_BYTES
    none = torch.empty(0, dtype=torch.uint8, device=DEV)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
    if fused:
        pkv.decode_step(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache, w.v_cache,
                        w.block_tables, w.decode_lens, w.rope_theta, w.scale, out,
                        workspace=none, partition_tokens=P)
    else:
        pkv.kv_append(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache, w.v_cache,
                      w.rope_theta)
        pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                   w.scale, out, workspace=none, partition_tokens=P)
    torch.cuda.synchronize()
    check_decode(out.cpu(), ref, torch.bfloat16, "static schedule")


@pytest.mark.parametrize("dtype,d,G", [(torch.bfloat16, 64, 4), (torch.bfloat16, 64, 8),
                                       (torch.bfloat16, 128, 4), (torch.float32, 64, 2),
                                       (torch.bfloat16, 64, 1)])
@pytest.mark.parametrize("P", [304, 1040])
@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "one_launch"])
def test_cluster_merge(dtype, d, G, P, fused):
    """Small batches: each (sequence, kv head) runs as one thread-block
    cluster, one partition per CTA, merged through distributed shared memory.
    The workspace partials stay untouched (no combine), sequences shorter
    than the cluster leave CTAs idle, and the result matches the oracle; with
    cluster=False the same call goes through the partials and the combine."""
    Hkv = 2
    lens = [2200, 15, 300, 1200]
    results = {}
    for cluster in (True, False):
        w = W.build_workload("cluster", lens, G * Hkv, Hkv, d, dtype, 1e4, seed=200 + d + G,
                             device=DEV, pool_factor=1.2)
        if not fused:
            w.decode_lens[1] = 0  # an empty context: all-zero output
        NP = -(-w.max_blocks * w.block_size // P)
        assert 2 <= NP <= 16
        assert pkv.decode_launches(w.B, w.Hq, w.Hkv, w.d, w.max_blocks, kv_dtype=dtype,
                                   out_dtype=torch.float32, partition_tokens=P, cluster=cluster,
                                   fused=fused) == (1 if cluster else 2)
        sub = SubProblem(w, range(w.B))
        need = pkv.decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks, kv_dtype=dtype,
                                         partition_tokens=P)
        ws = pkv.new_workspace(need, DEV)
        ws[pkv.SCHED_BYTES:].fill_(0x7F)
        out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
        if fused:
            pkv.decode_step(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache,
                            w.v_cache, w.block_tables, w.decode_lens, w.rope_theta, w.scale, out,
                            workspace=ws, partition_tokens=P, cluster=cluster)
        else:
            pkv.kv_append(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache,
                          w.v_cache, w.rope_theta)
            pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                       w.scale, out, workspace=ws, partition_tokens=P,
                                       cluster=cluster)
        torch.cuda.synchronize()
        partials_untouched = bool((ws[pkv.SCHED_BYTES:] == 0x7F).all())
        assert partials_untouched == cluster, f"cluster={cluster}: partials untouched={partials_untouched}"
        assert not ws[:pkv.SCHED_BYTES].any()
        _, _, _, ref = sub.oracle_step()
        if not fused:
            ref[1].zero_()
            assert not out[1].any()
        check_decode(out, ref, dtype, f"{dtype} d{d} G{G} P={P} fused={fused} cluster={cluster}")
        results[cluster] = out
    assert (results[True] - results[False]).abs().max().item() < 1e-4


def test_batch1_auto_partition_uses_clusters():
    """The batch-1 Llama-shaped step: the automatic partition cuts each kv
    head's context into 2..16 partitions that run as one cluster (one
    launch), and the result matches the oracle."""
    w = W.make_config(2, device=DEV)
    P = pkv.decode_partition_tokens(w.B, w.Hq, w.Hkv, w.d, w.max_blocks, kv_dtype=w.dtype)
    NP = -(-w.max_blocks * w.block_size // P)
    assert 2 <= NP <= 16
    assert pkv.decode_launches(w.B, w.Hq, w.Hkv, w.d, w.max_blocks, kv_dtype=w.dtype,
                               fused=True) == 1
    sub = SubProblem(w, range(w.B))
    out = gpu_step(w, out_dtype=torch.float32, fused=True)
    torch.cuda.synchronize()
    _, _, _, ref = sub.oracle_step()
    check_decode(out, ref, w.dtype, "batch-1 cluster step")


def test_prepared_decode_step_matches_decode_step():
    """prepare_decode_step marshals once; each call relaunches the step on the
    buffers' current contents: bit-identical to decode_step, also after q
    and the new rows change between calls."""
    w = W.build_workload("prepared", [300, 17, 2048, 64], 32, 8, 64, torch.bfloat16, 5e5,
                         seed=61, device=DEV)
    need = pkv.decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks)
    ws = pkv.new_workspace(need, DEV)
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    q = w.q.clone()
    out_p = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
    step = pkv.prepare_decode_step(q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache,
                                   w.v_cache, w.block_tables, w.decode_lens, w.rope_theta,
                                   w.scale, out_p, workspace=ws)
    g = torch.Generator(device=DEV)
    g.manual_seed(62)
    for rep in range(2):
        if rep:
            q.copy_(torch.randn(q.shape, generator=g, device=DEV).to(q.dtype))
        w.k_cache.copy_(k0)
        w.v_cache.copy_(v0)
        step()
        torch.cuda.synchronize()
        got = out_p.clone()
        w.k_cache.copy_(k0)
        w.v_cache.copy_(v0)
        out = torch.empty_like(out_p)
        pkv.decode_step(q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache, w.v_cache,
                        w.block_tables, w.decode_lens, w.rope_theta, w.scale, out, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(got, out), f"prepared call differs (rep {rep})"
