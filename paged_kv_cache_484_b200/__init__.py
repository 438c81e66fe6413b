"""B200-native (sm_100a) decode step over a paged KV cache.

The product is the C-ABI CUDA library ``_lib/libpkv.so`` (declared in
``include/pkv.h``); this package is its thin Python binding with the same
operation names:

* ``kv_append(q, k_new, v_new, positions, slot_mapping, k_cache, v_cache, rope_theta, stream)``
* ``paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, stream)``

plus ``decode_step`` (both in one launch), ``paged_attention_decode_noalloc``
and ``decode_workspace_size`` / ``decode_partition_tokens`` / ``new_workspace``
for planning.
PyTorch is used for device memory and streams only; the library is loaded on
first use and its absence is an error, never a fallback.
"""
from ._binding import (  # noqa: F401
    BLOCK_SIZE,
    BlockManager,
    DEVERR_BLOCK_ID,
    DEVERR_CONTEXT_LEN,
    DEVERR_PREFIX,
    DEVERR_SLOT,
    DEVERR_TIMEOUT,
    LIB_PATH,
    NOALLOC_SCRATCH_BYTES,
    PkvError,
    SCHED_BYTES,
    decode_launches,
    decode_partition_tokens,
    decode_step,
    decode_step_e4m3,
    prepare_decode_step,
    prepare_decode_step_e4m3,
    PreparedCall,
    decode_workspace_size,
    get_device_error,
    selftest_bounded_wait,
    PKV_ERR_DEVICE,
    kv_admission_capacity,
    kv_append,
    kv_append_e4m3,
    kv_request_bytes,
    load_library,
    new_workspace,
    paged_attention_decode,
    paged_attention_decode_cascade,
    paged_attention_decode_e4m3,
    paged_attention_decode_noalloc,
    decode_cascade_workspace_size,
    paged_attention_prefill,
    prefill_partition_tokens,
    prefill_workspace_size,
    version,
)
