"""The allocation-free decode entry point (GPU only).

pkv_paged_attention_decode_noalloc serves callers that cannot give the
library a workspace -- for example an engine that has reserved nearly all
device memory for its KV block pool, or a plugin interface that passes only
inputs and outputs.  It keeps the split-context scratch in the library's own
per-GPU array instead.  These tests call it through the C ABI and check that
its output matches the workspace-taking entry point on two calls in a row
(the second with different inputs, so leftovers from the first would show),
and that shapes needing more scratch than the array holds are refused before
any launch.  This file is collected last on purpose.
"""
from __future__ import annotations

import pytest
import torch

import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL_BF16 = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _both(w, P):
    """Output of the workspace entry point and of the allocation-free one."""
    ref = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=DEV)
    pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens, w.scale,
                               ref, partition_tokens=P)
    got = torch.full_like(ref, float("nan"))
    pkv.paged_attention_decode_noalloc(w.q, w.k_cache, w.v_cache, w.block_tables, w.decode_lens,
                                       w.scale, got, partition_tokens=P)
    torch.cuda.synchronize()
    return ref, got


@pytest.mark.parametrize("d,G,P", [(64, 4, 64), (128, 8, 256), (64, 1, 0)])
def test_matches_workspace_entry_point_twice(d, G, P):
    Hkv = 2
    first = W.build_workload("noalloc-a", [2999, 17, 640, 0, 1500], G * Hkv, Hkv, d,
                             torch.bfloat16, 5e5, seed=31 + d + G, device=DEV)
    second = W.build_workload("noalloc-b", [700, 3100, 5, 1023], G * Hkv, Hkv, d,
                              torch.bfloat16, 5e5, seed=37 + d + G, device=DEV)
    for w in (first, second):
        need = pkv.decode_workspace_size(w.B, w.Hq, w.Hkv, w.d, w.max_blocks,
                                         partition_tokens=P)
        assert need <= pkv.NOALLOC_SCRATCH_BYTES
        ref, got = _both(w, P)
        assert torch.isfinite(got).all()
        assert (got - ref).abs().max().item() <= TOL_BF16


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
