"""The allocation-free decode entry point (GPU only).

pkv_paged_attention_decode_noalloc serves callers that cannot give the
library a workspace -- for example an engine that has reserved nearly all
device memory for its KV block pool, or a plugin interface that passes only
inputs and outputs.  It keeps the split-context scratch in the library's own
per-GPU array instead.  These tests call it through the C ABI and check that
its output equals, bit for bit, the workspace-taking entry point's (the two
run the same plan and kernels) on two calls in a row (the second with
different inputs, so leftovers from the first would show), with and without
thread-block-cluster merging (without it the scheduler's counters in the
built-in array are used); that both agree with the fp64 oracle on host
copies of the inputs; and that shapes needing more scratch than the array
holds are refused before any launch.  This file is collected last on
purpose.
"""
from __future__ import annotations

import pytest
import torch

import oracle
import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200 import workloads as W
from paged_kv_cache_484_b200.workloads import extract_sequences

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL_BF16 = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _both(w, P, cluster):
    """Output of the workspace entry point and of the allocation-free one."""
    ref = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
    pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens, w.scale,
                               ref, partition_tokens=P, cluster=cluster)
    got = torch.full_like(ref, float("nan"))
    pkv.paged_attention_decode_noalloc(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                       w.scale, got, partition_tokens=P, cluster=cluster)
    torch.cuda.synchronize()
    return ref, got


@pytest.mark.parametrize("d,G,P,cluster", [(64, 4, 64, True), (128, 8, 256, True),
                                           (64, 1, 0, True), (64, 4, 64, False),
                                           (128, 4, 128, False)])
def test_matches_workspace_entry_point_twice(d, G, P, cluster):
    Hkv = 2
    first = W.build_workload("noalloc-a", [2999, 17, 640, 0, 1500], G * Hkv, Hkv, d,
                             torch.bfloat16, 5e5, seed=31 + d + G, device=DEV)
    second = W.build_workload("noalloc-b", [700, 3100, 5, 1023], G * Hkv, Hkv, d,
                              torch.bfloat16, 5e5, seed=37 + d + G, device=DEV)
    for w in (first, second):
        need = pkv.decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks,
                                         partition_tokens=P)
        assert need <= pkv.NOALLOC_SCRATCH_BYTES
        # the oracle's inputs, copied to the host before any library call
        sub = extract_sequences(w, range(w.B))
        ref, got = _both(w, P, cluster)
        assert torch.isfinite(got).all()
        # the same plan and kernels as the workspace entry point: equal bits
        assert torch.equal(got, ref)
        want = oracle.paged_attention_decode(sub.q, sub.k_cache, sub.v_cache, sub.tables,
                                             sub.decode_lens, sub.scale, nthreads=8)
        assert (got.double().cpu() - want).abs().max().item() <= TOL_BF16


def test_refuses_shapes_beyond_the_builtin_scratch():
    # 64 sequences of up to 8192 tokens split into 16-token partitions would
    # need far more than the built-in scratch: refused before any launch
    w = W.build_workload("noalloc-big", [8191] * 64, 8, 2, 64, torch.bfloat16, 5e5, seed=41,
                         device=DEV)
    need = pkv.decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks, partition_tokens=16)
    assert need > pkv.NOALLOC_SCRATCH_BYTES
    out = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(pkv.PkvError) as exc:
        pkv.paged_attention_decode_noalloc(w.q, w.k_cache, w.v_cache, w.block_tables,
                                           w.decode_lens, w.scale, out, partition_tokens=16)
    assert exc.value.status == 3
    torch.cuda.synchronize()
    assert not out.any()
