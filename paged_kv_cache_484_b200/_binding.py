"""ctypes marshalling for the C ABI in include/pkv.h.

Every function here only checks tensor metadata, turns tensors into raw
device pointers plus sizes, and calls the library; all arithmetic of the
decode step runs in the CUDA kernels of ``_lib/libpkv.so``.  If that library
is missing the call raises -- there is no fallback path.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libpkv.so")

PKV_DTYPE_F32 = 0
PKV_DTYPE_BF16 = 1
PKV_DTYPE_E4M3 = 2  # 8-bit cache (uint8 tensors of E4M3 codes)
PKV_DECODE_FORCE_SIMT = 0x1
PKV_DECODE_NO_CLUSTER = 0x2
DEVERR_SLOT = 0x1
DEVERR_BLOCK_ID = 0x2
DEVERR_CONTEXT_LEN = 0x4
DEVERR_TIMEOUT = 0x8
DEVERR_PREFIX = 0x10
BLOCK_SIZE = 16
NOALLOC_SCRATCH_BYTES = 16 << 20   # PKV_NOALLOC_SCRATCH_BYTES in include/pkv.h

_lock = threading.Lock()
_lib = None


class PkvError(RuntimeError):
    """A non-OK status from the C ABI (``status`` holds the pkv_status code)."""

    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


def load_library() -> ctypes.CDLL:
    """Load libpkv.so (built by ``paged_kv_cache_484_b200.build``); raise if absent."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"CUDA library {LIB_PATH} is not built; run "
                "`python -m paged_kv_cache_484_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32
        lib.pkv_kv_append.argtypes = [vp, vp, vp, vp, vp, vp, vp,
                                      i64, i64, i64, i64, i64, i64, i32, ctypes.c_double, vp, vp]
        lib.pkv_kv_append.restype = ctypes.c_int
        lib.pkv_decode_workspace_size.argtypes = [i64, i64, i64, i64, i64, i64, i32, i32]
        lib.pkv_decode_workspace_size.restype = ctypes.c_size_t
        lib.pkv_decode_launches.argtypes = [i64, i64, i64, i64, i64, i64, i32, i32, i32, u32, i32]
        lib.pkv_decode_launches.restype = i32
        lib.pkv_decode_partition_tokens.argtypes = [i64, i64, i64, i64, i64, i64, i32]
        lib.pkv_decode_partition_tokens.restype = i32
        lib.pkv_paged_attention_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                                   i64, i64, i64, i64, i64, i64, i64,
                                                   i32, i32, ctypes.c_float, i32, u32, vp, vp]
        lib.pkv_paged_attention_decode.restype = ctypes.c_int
        lib.pkv_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                        ctypes.c_size_t, i64, i64, i64, i64, i64, i64, i64,
                                        i32, i32, ctypes.c_double, ctypes.c_float, i32, u32,
                                        vp, vp]
        lib.pkv_decode_step.restype = ctypes.c_int
        lib.pkv_decode_step_window.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                               ctypes.c_size_t, i64, i64, i64, i64, i64, i64,
                                               i64, i32, i32, ctypes.c_double, ctypes.c_float,
                                               i32, i32, u32, vp, vp]
        lib.pkv_decode_step_window.restype = ctypes.c_int
        lib.pkv_paged_attention_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, vp,
                                                           i64, i64, i64, i64, i64, i64, i64,
                                                           i32, i32, ctypes.c_float, i32, u32,
                                                           vp, vp]
        lib.pkv_paged_attention_decode_noalloc.restype = ctypes.c_int
        lib.pkv_paged_attention_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                                     i64, i64, i64, i64, i64, i64, i64, i64,
                                                     i32, i32, ctypes.c_float, i32, i32, vp, vp]
        lib.pkv_paged_attention_prefill.restype = ctypes.c_int
        lib.pkv_prefill_workspace_size.argtypes = [i64, i64, i64, i64, i64, i64, i64, i32]
        lib.pkv_prefill_workspace_size.restype = ctypes.c_size_t
        lib.pkv_prefill_partition_tokens.argtypes = [i64, i64, i64, i64, i64, i64, i64]
        lib.pkv_prefill_partition_tokens.restype = i32
        lib.pkv_paged_attention_decode_cascade.argtypes = [
            vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i64, i64, i64, i64, i64, i64,
            i64, i64, i64, i32, i32, ctypes.c_float, i32, u32, vp, vp]
        lib.pkv_paged_attention_decode_cascade.restype = ctypes.c_int
        lib.pkv_paged_attention_decode_cascade_window.argtypes = [
            vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i64, i64, i64, i64, i64, i64,
            i64, i64, i64, i32, i32, ctypes.c_float, i32, i32, u32, vp, vp]
        lib.pkv_paged_attention_decode_cascade_window.restype = ctypes.c_int
        lib.pkv_decode_cascade_workspace_size.argtypes = [i64, i64, i64, i64, i64, i64, i32, i32]
        lib.pkv_decode_cascade_workspace_size.restype = ctypes.c_size_t
        lib.pkv_kv_append_e4m3.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                           i64, i32, ctypes.c_double, ctypes.c_float,
                                           ctypes.c_float, vp, vp]
        lib.pkv_kv_append_e4m3.restype = ctypes.c_int
        lib.pkv_paged_attention_decode_e4m3.argtypes = [
            vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i64, i64, i64, i64, i64, i64, i64, i32,
            ctypes.c_float, ctypes.c_float, ctypes.c_float, i32, i32, u32, vp, vp]
        lib.pkv_paged_attention_decode_window.argtypes = [
            vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i64, i64, i64, i64, i64, i64, i64, i32,
            i32, ctypes.c_float, i32, i32, u32, vp, vp]
        lib.pkv_paged_attention_decode_window.restype = ctypes.c_int
        lib.pkv_paged_attention_decode_e4m3.restype = ctypes.c_int
        lib.pkv_decode_step_e4m3.argtypes = [
            vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i64, i64, i64, i64, i64,
            i64, i64, i32, ctypes.c_double, ctypes.c_float, ctypes.c_float, ctypes.c_float, i32,
            i32, u32, vp, vp]
        lib.pkv_decode_step_e4m3.restype = ctypes.c_int
        lib.pkv_kv_request_bytes.argtypes = [i64, i64, i64, i64, i64, i32]
        lib.pkv_kv_request_bytes.restype = i64
        lib.pkv_kv_admission_capacity.argtypes = [i64, i64, i64, i64, i64, i64, i32]
        lib.pkv_kv_admission_capacity.restype = i64
        lib.pkv_bm_create.argtypes = [i32, i32]
        lib.pkv_bm_create.restype = vp
        lib.pkv_bm_destroy.argtypes = [vp]
        lib.pkv_bm_destroy.restype = None
        lib.pkv_bm_add_sequence.argtypes = [vp, i64, vp, i64, vp]
        lib.pkv_bm_add_sequence.restype = ctypes.c_int
        lib.pkv_bm_prompt_slots.argtypes = [vp, i64, vp, i64]
        lib.pkv_bm_prompt_slots.restype = ctypes.c_int
        lib.pkv_bm_append.argtypes = [vp, i64, i32, vp]
        lib.pkv_bm_append.restype = ctypes.c_int
        lib.pkv_bm_free_sequence.argtypes = [vp, i64]
        lib.pkv_bm_free_sequence.restype = ctypes.c_int
        lib.pkv_bm_block_table.argtypes = [vp, i64, vp, i32, vp, vp]
        lib.pkv_bm_block_table.restype = ctypes.c_int
        lib.pkv_bm_shared_tokens.argtypes = [vp, i64]
        lib.pkv_bm_shared_tokens.restype = i32
        lib.pkv_bm_free_blocks.argtypes = [vp]
        lib.pkv_bm_free_blocks.restype = i32
        lib.pkv_bm_cached_blocks.argtypes = [vp]
        lib.pkv_bm_cached_blocks.restype = i32
        lib.pkv_status_string.argtypes = [i32]
        lib.pkv_status_string.restype = ctypes.c_char_p
        lib.pkv_last_error.argtypes = []
        lib.pkv_last_error.restype = ctypes.c_char_p
        lib.pkv_version.argtypes = []
        lib.pkv_version.restype = i32
        lib.pkv_get_device_error.argtypes = [vp, vp, vp]
        lib.pkv_get_device_error.restype = ctypes.c_int
        lib.pkv_selftest_bounded_wait.argtypes = [u32, vp, vp, vp]
        lib.pkv_selftest_bounded_wait.restype = ctypes.c_int
        _lib = lib
        return lib


def _raise(status: int, lib, what: str):
    if status != 0:
        detail = lib.pkv_last_error().decode()
        raise PkvError(status, f"{what}: {lib.pkv_status_string(status).decode()}"
                               + (f" ({detail})" if detail else ""))


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return PKV_DTYPE_F32
    if dt == torch.bfloat16:
        return PKV_DTYPE_BF16
    raise TypeError(f"unsupported dtype {dt} (float32 or bfloat16)")


def _kv_dtype_code(dt: torch.dtype) -> int:
    """Cache dtype code: float32, bfloat16, or uint8 for the 8-bit cache."""
    if dt == torch.uint8:
        return PKV_DTYPE_E4M3
    return _dtype_code(dt)


def _dev(t: torch.Tensor, name: str, dtype=None, on=None) -> int:
    """Device address of a contiguous CUDA tensor.  ``on``: the device of the
    call (that of q); a kernel may only be handed memory of its own GPU."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if on is not None and t.device != on:
        raise ValueError(f"{name} is on {t.device}, the call's other tensors on {on}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


@contextlib.contextmanager
def _current(dv: torch.device):
    """Makes the call's device (that of q) the current CUDA device for one
    library call: the library plans a launch from the current device's SM
    count and shared-memory limit, and the allocation-free decode looks up
    its built-in scratch on the current device, while the kernels run on the
    stream of the call's device."""
    if dv.type == "cuda" and torch.cuda.is_available() and \
            torch.cuda.current_device() != dv.index:
        with torch.cuda.device(dv):
            yield
    else:
        yield


def _flags(force_simt: bool, cluster: bool) -> int:
    return (PKV_DECODE_FORCE_SIMT if force_simt else 0) | (0 if cluster else PKV_DECODE_NO_CLUSTER)


def _stream_ptr(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def kv_append(q, k_new, v_new, positions, slot_mapping, k_cache, v_cache, rope_theta,
              stream=None, *, device_error=None) -> None:
    """RoPE on q (in place) and k_new; write k and v into their cache slots.

    q [T, Hq, d], k_new/v_new [T, Hkv, d], k_cache/v_cache [NB, Hkv, 16, d]
    (one dtype, float32 or bfloat16), positions/slot_mapping int64 [T]
    (slot < 0: skip the write).  See include/pkv.h, pkv_kv_append.
    """
    lib = load_library()
    dv = q.device
    dt = _dtype_code(q.dtype)
    for name, t in (("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache), ("v_cache", v_cache)):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from q dtype {q.dtype}")
    T, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if k_new.shape != (T, Hkv, d) or v_new.shape != (T, Hkv, d) or v_cache.shape != k_cache.shape \
            or d2 != d or positions.shape != (T,) or slot_mapping.shape != (T,):
        raise ValueError("inconsistent kv_append shapes")
    err = (_dev(device_error, "device_error", torch.int32, on=dv)
           if device_error is not None else None)
    with _current(dv):
        st = lib.pkv_kv_append(
            _dev(q, "q", on=dv), _dev(k_new, "k_new", on=dv), _dev(v_new, "v_new", on=dv),
            _dev(positions, "positions", torch.int64, on=dv),
            _dev(slot_mapping, "slot_mapping", torch.int64, on=dv),
            _dev(k_cache, "k_cache", on=dv), _dev(v_cache, "v_cache", on=dv),
            T, Hq, Hkv, d, NB, bs, dt, float(rope_theta), err, _stream_ptr(stream, q.device))
    _raise(st, lib, "kv_append")


def decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                            kv_dtype=torch.bfloat16, block_size=BLOCK_SIZE) -> int:
    """Partition length the decode call picks when ``partition_tokens`` is 0."""
    lib = load_library()
    return int(lib.pkv_decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                               max_blocks_per_seq, block_size,
                                               _kv_dtype_code(kv_dtype)))


def decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                          kv_dtype=torch.bfloat16, partition_tokens=0,
                          block_size=BLOCK_SIZE) -> int:
    """Bytes of workspace ``paged_attention_decode`` needs for these shapes."""
    lib = load_library()
    return int(lib.pkv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                             max_blocks_per_seq, block_size,
                                             _kv_dtype_code(kv_dtype), int(partition_tokens)))


def decode_launches(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                    kv_dtype=torch.bfloat16, out_dtype=torch.bfloat16, partition_tokens=0,
                    force_simt=False, cluster=True, fused=False, block_size=BLOCK_SIZE) -> int:
    """Kernels one decode call with these shapes launches on the current
    device: 1 (no split, or split contexts merged inside thread-block
    clusters) or 2 (decode + partition combine); 0 for invalid arguments."""
    lib = load_library()
    return int(lib.pkv_decode_launches(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                       max_blocks_per_seq, block_size, _kv_dtype_code(kv_dtype),
                                       _dtype_code(out_dtype), int(partition_tokens),
                                       _flags(force_simt, cluster), 1 if fused else 0))


SCHED_BYTES = 256  # scheduler counters at the head of a decode workspace


def new_workspace(nbytes, device) -> torch.Tensor:
    """A decode workspace of ``nbytes`` on ``device`` with its scheduler
    counters zeroed (the rest needs no initialisation); reusable by later
    calls, which leave the counters zero."""
    ws = torch.empty(max(int(nbytes), SCHED_BYTES), dtype=torch.uint8, device=device)
    ws[:SCHED_BYTES].zero_()
    return ws


def paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out,
                           stream=None, *, workspace=None, partition_tokens=0, force_simt=False,
                           device_error=None, cluster=True, sliding_window=0) -> torch.Tensor:
    """Single-query attention over the paged cache; writes and returns ``out``.

    q [B, Hq, d] and caches [NB, Hkv, 16, d] share a dtype (float32 or
    bfloat16); block_tables int32 [B, MB]; context_lens int32 [B];
    out [B, Hq, d] float32 or bfloat16.  ``workspace`` (uint8 CUDA tensor of
    at least ``decode_workspace_size`` bytes, see ``new_workspace``) is
    allocated from PyTorch's caching allocator when not given; an empty tensor
    passes none, which is allowed when no context is split (the work items
    are then dealt out round-robin).  ``sliding_window`` > 0: each query
    attends to the last ``sliding_window`` tokens of its context
    (pkv_paged_attention_decode_window).  See include/pkv.h.
    """
    lib = load_library()
    dv = q.device
    kv_dt = _dtype_code(k_cache.dtype)
    if q.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share one dtype")
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if v_cache.shape != k_cache.shape or d2 != d or out.shape != (B, Hq, d) \
            or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("inconsistent paged_attention_decode shapes")
    out_dt = _dtype_code(out.dtype)
    if workspace is None:
        need = lib.pkv_decode_workspace_size(B, Hq, Hkv, d, MB, bs, kv_dt, int(partition_tokens))
        workspace = new_workspace(int(need), q.device)
    err = (_dev(device_error, "device_error", torch.int32, on=dv)
           if device_error is not None else None)
    args = [_dev(q, "q", on=dv), _dev(k_cache, "k_cache", on=dv), _dev(v_cache, "v_cache", on=dv),
            _dev(block_tables, "block_tables", torch.int32, on=dv),
            _dev(context_lens, "context_lens", torch.int32, on=dv), _dev(out, "out", on=dv),
            _dev(workspace, "workspace", on=dv), workspace.numel() * workspace.element_size(),
            B, Hq, Hkv, d, NB, bs, MB, kv_dt, out_dt, float(scale)]
    tail = [int(partition_tokens), _flags(force_simt, cluster), err, _stream_ptr(stream, q.device)]
    if sliding_window:
        with _current(dv):
            st = lib.pkv_paged_attention_decode_window(*args, int(sliding_window), *tail)
    else:
        with _current(dv):
            st = lib.pkv_paged_attention_decode(*args, *tail)
    _raise(st, lib, "paged_attention_decode")
    return out


def kv_append_e4m3(q, k_new, v_new, positions, slot_mapping, kv_cache, rope_theta,
                   k_scale, v_scale, stream=None, *, device_error=None) -> None:
    """``kv_append`` into the 8-bit cache: q [T, Hq, d] rotated in place (its
    own dtype, float32 or bfloat16, shared by k_new/v_new [T, Hkv, d]);
    kv_cache uint8 [NB, Hkv, 2, 16 * d]: each page's K half [16][d] gets the
    E4M3 codes of rope(k) / k_scale, its V half [d][16] (transposed) those of
    v / v_scale.  See include/pkv.h, pkv_kv_append_e4m3."""
    lib = load_library()
    dv = q.device
    dt = _dtype_code(q.dtype)
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from q dtype {q.dtype}")
    T, Hq, d = q.shape
    if kv_cache.dim() != 4:
        raise ValueError("kv_cache must be [num_blocks, Hkv, 2, 16 * head_dim]")
    NB, Hkv, two, pg = kv_cache.shape
    bs = BLOCK_SIZE
    if k_new.shape != (T, Hkv, d) or v_new.shape != (T, Hkv, d) or two != 2 or pg != bs * d \
            or positions.shape != (T,) or slot_mapping.shape != (T,):
        raise ValueError("inconsistent kv_append_e4m3 shapes")
    err = (_dev(device_error, "device_error", torch.int32, on=dv)
           if device_error is not None else None)
    with _current(dv):
        st = lib.pkv_kv_append_e4m3(
            _dev(q, "q", on=dv), _dev(k_new, "k_new", on=dv), _dev(v_new, "v_new", on=dv),
            _dev(positions, "positions", torch.int64, on=dv),
            _dev(slot_mapping, "slot_mapping", torch.int64, on=dv),
            _dev(kv_cache, "kv_cache", torch.uint8, on=dv),
            T, Hq, Hkv, d, NB, bs, dt, float(rope_theta), float(k_scale), float(v_scale), err,
            _stream_ptr(stream, q.device))
    _raise(st, lib, "kv_append_e4m3")


def paged_attention_decode_e4m3(q, kv_cache, block_tables, context_lens, scale, k_scale,
                                v_scale, out, stream=None, *, workspace=None, partition_tokens=0,
                                device_error=None, cluster=True,
                                sliding_window=0) -> torch.Tensor:
    """``paged_attention_decode`` over the 8-bit cache (kv_cache uint8
    [NB, Hkv, 2, 16 * d]: per page its K half [16][d], then its V half
    [d][16]); q bfloat16 [B, Hq, d]; cached values are code x k_scale /
    code x v_scale.  Writes and returns ``out`` (float32 or bfloat16).  See
    include/pkv.h."""
    lib = load_library()
    dv = q.device
    B, Hq, d = q.shape
    if kv_cache.dim() != 4:
        raise ValueError("kv_cache must be [num_blocks, Hkv, 2, 16 * head_dim]")
    NB, Hkv, two, pg = kv_cache.shape
    bs = BLOCK_SIZE
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if two != 2 or pg != bs * d or out.shape != (B, Hq, d) \
            or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("inconsistent paged_attention_decode_e4m3 shapes")
    if workspace is None:
        need = lib.pkv_decode_workspace_size(B, Hq, Hkv, d, MB, bs, PKV_DTYPE_E4M3,
                                             int(partition_tokens))
        workspace = new_workspace(int(need), q.device)
    err = (_dev(device_error, "device_error", torch.int32, on=dv)
           if device_error is not None else None)
    with _current(dv):
        st = lib.pkv_paged_attention_decode_e4m3(
            _dev(q, "q", torch.bfloat16, on=dv), _dev(kv_cache, "kv_cache", torch.uint8, on=dv),
            _dev(block_tables, "block_tables", torch.int32, on=dv),
            _dev(context_lens, "context_lens", torch.int32, on=dv), _dev(out, "out", on=dv),
            _dev(workspace, "workspace", on=dv), workspace.numel() * workspace.element_size(),
            B, Hq, Hkv, d, NB, bs, MB, _dtype_code(out.dtype), float(scale), float(k_scale),
            float(v_scale), int(sliding_window), int(partition_tokens), _flags(False, cluster), err,
            _stream_ptr(stream, q.device))
    _raise(st, lib, "paged_attention_decode_e4m3")
    return out


def _decode_step_args(q, k_new, v_new, positions, slot_mapping, k_cache, v_cache, block_tables,
                      context_lens, rope_theta, scale, out, stream, workspace, partition_tokens,
                      force_simt, device_error, cluster):
    """Checked pkv_decode_step arguments (allocating a workspace if none is
    given), and the tensors they point into."""
    lib = load_library()
    dv = q.device
    kv_dt = _dtype_code(k_cache.dtype)
    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("v_cache", v_cache)):
        if t.dtype != k_cache.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from the cache dtype {k_cache.dtype}")
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if v_cache.shape != k_cache.shape or d2 != d or out.shape != (B, Hq, d) \
            or k_new.shape != (B, Hkv, d) or v_new.shape != (B, Hkv, d) \
            or positions.shape != (B,) or slot_mapping.shape != (B,) \
            or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("inconsistent decode_step shapes")
    if workspace is None:
        need = lib.pkv_decode_workspace_size(B, Hq, Hkv, d, MB, bs, kv_dt, int(partition_tokens))
        workspace = new_workspace(int(need), q.device)
    err = (_dev(device_error, "device_error", torch.int32, on=dv)
           if device_error is not None else None)
    args = (_dev(q, "q", on=dv), _dev(k_new, "k_new", on=dv), _dev(v_new, "v_new", on=dv),
            _dev(positions, "positions", torch.int64, on=dv),
            _dev(slot_mapping, "slot_mapping", torch.int64, on=dv),
            _dev(k_cache, "k_cache", on=dv), _dev(v_cache, "v_cache", on=dv),
            _dev(block_tables, "block_tables", torch.int32, on=dv),
            _dev(context_lens, "context_lens", torch.int32, on=dv), _dev(out, "out", on=dv),
            _dev(workspace, "workspace", on=dv), workspace.numel() * workspace.element_size(),
            B, Hq, Hkv, d, NB, bs, MB, kv_dt, _dtype_code(out.dtype), float(rope_theta),
            float(scale), int(partition_tokens), _flags(force_simt, cluster), err,
            _stream_ptr(stream, q.device))
    keep = (q, k_new, v_new, positions, slot_mapping, k_cache, v_cache, block_tables,
            context_lens, out, workspace, device_error)
    return lib, args, keep


def decode_step(q, k_new, v_new, positions, slot_mapping, k_cache, v_cache, block_tables,
                context_lens, rope_theta, scale, out, stream=None, *, workspace=None,
                partition_tokens=0, force_simt=False, device_error=None,
                cluster=True, sliding_window=0) -> torch.Tensor:
    """``kv_append`` (one new token per sequence) then ``paged_attention_decode``,
    in one launch.  The new token must be the last token of its context
    (context_lens[b] - 1, at the slot block_tables gives it).  q is read only:
    the rotated q is used inside the kernel and not stored.  ``sliding_window``
    > 0: each query attends to the last ``sliding_window`` tokens of its context
    (pkv_decode_step_window).  See include/pkv.h, pkv_decode_step.
    """
    lib, args, _ = _decode_step_args(q, k_new, v_new, positions, slot_mapping, k_cache, v_cache,
                                     block_tables, context_lens, rope_theta, scale, out, stream,
                                     workspace, partition_tokens, force_simt, device_error,
                                     cluster)
    with _current(q.device):
        if sliding_window:
            # pkv_decode_step_window takes the window just before partition_tokens
            st = lib.pkv_decode_step_window(*args[:-4], int(sliding_window), *args[-4:])
        else:
            st = lib.pkv_decode_step(*args)
    _raise(st, lib, "decode_step")
    return out


class PreparedCall:
    """A library call whose arguments were checked and marshalled once.
    Calling it launches the same work again on the same stream; the tensors
    it was prepared with must stay alive and keep their shapes, dtypes and
    addresses (their contents may change between calls)."""

    __slots__ = ("_lib", "_fn", "_args", "_name", "_keep", "_dev")

    def __init__(self, lib, fn, args, name, keep, device=None):
        self._lib, self._fn, self._name, self._keep = lib, fn, name, keep
        self._dev = device
        types = fn.argtypes
        # ctypes instances, so that a call converts nothing
        self._args = tuple(t(a) if a is not None or t is not ctypes.c_void_p else t()
                           for t, a in zip(types, args))

    def __call__(self) -> None:
        if self._dev is not None:
            with _current(self._dev):
                st = self._fn(*self._args)
        else:
            st = self._fn(*self._args)
        if st != 0:
            _raise(st, self._lib, self._name)


def prepare_decode_step(q, k_new, v_new, positions, slot_mapping, k_cache, v_cache, block_tables,
                        context_lens, rope_theta, scale, out, stream=None, *, workspace,
                        partition_tokens=0, force_simt=False, device_error=None,
                        cluster=True) -> PreparedCall:
    """``decode_step`` checked and marshalled once, for a caller that repeats
    the same step on the same buffers (a model's layer loop: one prepared call
    per layer).  ``workspace`` is required; see ``decode_step``."""
    lib, args, keep = _decode_step_args(q, k_new, v_new, positions, slot_mapping, k_cache,
                                        v_cache, block_tables, context_lens, rope_theta, scale,
                                        out, stream, workspace, partition_tokens, force_simt,
                                        device_error, cluster)
    return PreparedCall(lib, lib.pkv_decode_step, args, "decode_step", keep, q.device)


def _decode_step_e4m3_args(q, k_new, v_new, positions, slot_mapping, kv_cache, block_tables,
                           context_lens, rope_theta, scale, k_scale, v_scale, out, stream,
                           workspace, partition_tokens, device_error, cluster, sliding_window):
    """Checked pkv_decode_step_e4m3 arguments (allocating a workspace if none
    is given), and the tensors they point into."""
    lib = load_library()
    dv = q.device
    B, Hq, d = q.shape
    if kv_cache.dim() != 4:
        raise ValueError("kv_cache must be [num_blocks, Hkv, 2, 16 * head_dim]")
    NB, Hkv, two, pg = kv_cache.shape
    bs = BLOCK_SIZE
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if two != 2 or pg != bs * d or out.shape != (B, Hq, d) \
            or k_new.shape != (B, Hkv, d) or v_new.shape != (B, Hkv, d) \
            or positions.shape != (B,) or slot_mapping.shape != (B,) \
            or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("inconsistent decode_step_e4m3 shapes")
    if workspace is None:
        need = lib.pkv_decode_workspace_size(B, Hq, Hkv, d, MB, bs, PKV_DTYPE_E4M3,
                                             int(partition_tokens))
        workspace = new_workspace(int(need), q.device)
    err = (_dev(device_error, "device_error", torch.int32, on=dv)
           if device_error is not None else None)
    args = (_dev(q, "q", torch.bfloat16, on=dv), _dev(k_new, "k_new", torch.bfloat16, on=dv),
            _dev(v_new, "v_new", torch.bfloat16, on=dv),
            _dev(positions, "positions", torch.int64, on=dv),
            _dev(slot_mapping, "slot_mapping", torch.int64, on=dv),
            _dev(kv_cache, "kv_cache", torch.uint8, on=dv),
            _dev(block_tables, "block_tables", torch.int32, on=dv),
            _dev(context_lens, "context_lens", torch.int32, on=dv), _dev(out, "out", on=dv),
            _dev(workspace, "workspace", on=dv), workspace.numel() * workspace.element_size(),
            B, Hq, Hkv, d, NB, bs, MB, _dtype_code(out.dtype), float(rope_theta), float(scale),
            float(k_scale), float(v_scale), int(sliding_window), int(partition_tokens),
            _flags(False, cluster), err, _stream_ptr(stream, q.device))
    keep = (q, k_new, v_new, positions, slot_mapping, kv_cache, block_tables, context_lens, out,
            workspace, device_error)
    return lib, args, keep


def decode_step_e4m3(q, k_new, v_new, positions, slot_mapping, kv_cache, block_tables,
                     context_lens, rope_theta, scale, k_scale, v_scale, out, stream=None, *,
                     workspace=None, partition_tokens=0, device_error=None, cluster=True,
                     sliding_window=0) -> torch.Tensor:
    """``kv_append_e4m3`` (one new token per sequence, bfloat16 q/k_new/v_new)
    then ``paged_attention_decode_e4m3``, in one launch; the new codes equal
    the append's.  q is read only.  See include/pkv.h, pkv_decode_step_e4m3."""
    lib, args, _ = _decode_step_e4m3_args(q, k_new, v_new, positions, slot_mapping, kv_cache,
                                          block_tables, context_lens, rope_theta, scale, k_scale,
                                          v_scale, out, stream, workspace, partition_tokens,
                                          device_error, cluster, sliding_window)
    with _current(q.device):
        st = lib.pkv_decode_step_e4m3(*args)
    _raise(st, lib, "decode_step_e4m3")
    return out


def prepare_decode_step_e4m3(q, k_new, v_new, positions, slot_mapping, kv_cache, block_tables,
                             context_lens, rope_theta, scale, k_scale, v_scale, out, stream=None,
                             *, workspace, partition_tokens=0, device_error=None, cluster=True,
                             sliding_window=0) -> PreparedCall:
    """``decode_step_e4m3`` checked and marshalled once (see
    ``prepare_decode_step``)."""
    lib, args, keep = _decode_step_e4m3_args(q, k_new, v_new, positions, slot_mapping, kv_cache,
                                             block_tables, context_lens, rope_theta, scale,
                                             k_scale, v_scale, out, stream, workspace,
                                             partition_tokens, device_error, cluster,
                                             sliding_window)
    return PreparedCall(lib, lib.pkv_decode_step_e4m3, args, "decode_step_e4m3", keep, q.device)


def paged_attention_decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, scale, out,
                                   stream=None, *, partition_tokens=0, force_simt=False,
                                   device_error=None, cluster=True) -> torch.Tensor:
    """``paged_attention_decode`` for callers that cannot allocate device memory.

    Same arguments and result, but no workspace: the split-context scratch is
    the library's built-in per-GPU array of NOALLOC_SCRATCH_BYTES, shared by
    every call on the device (calls that overlap on the GPU race on it).
    Shapes that need more scratch raise PkvError (status 3) before any launch.
    See include/pkv.h, pkv_paged_attention_decode_noalloc.
    """
    lib = load_library()
    dv = q.device
    kv_dt = _dtype_code(k_cache.dtype)
    if q.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share one dtype")
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if v_cache.shape != k_cache.shape or d2 != d or out.shape != (B, Hq, d) \
            or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("inconsistent paged_attention_decode_noalloc shapes")
    err = (_dev(device_error, "device_error", torch.int32, on=dv)
           if device_error is not None else None)
    with _current(dv):
        st = lib.pkv_paged_attention_decode_noalloc(
            _dev(q, "q", on=dv), _dev(k_cache, "k_cache", on=dv), _dev(v_cache, "v_cache", on=dv),
            _dev(block_tables, "block_tables", torch.int32, on=dv),
            _dev(context_lens, "context_lens", torch.int32, on=dv), _dev(out, "out", on=dv),
            B, Hq, Hkv, d, NB, bs, MB, kv_dt, _dtype_code(out.dtype), float(scale),
            int(partition_tokens), _flags(force_simt, cluster), err,
            _stream_ptr(stream, q.device))
    _raise(st, lib, "paged_attention_decode_noalloc")
    return out


PKV_ERR_DEVICE = 5


def get_device_error(device_error, stream=None) -> int:
    """Wait for ``stream`` (default: the current stream of the word's device)
    and return the device error word (PKV_DEVERR_* bits; 0 = none).
    See include/pkv.h, pkv_get_device_error."""
    lib = load_library()
    dv = device_error.device
    code = ctypes.c_int32(0)
    with _current(dv):
        st = lib.pkv_get_device_error(_dev(device_error, "device_error", torch.int32),
                                      _stream_ptr(stream, dv), ctypes.byref(code))
    if st not in (0, PKV_ERR_DEVICE):
        _raise(st, lib, "get_device_error")
    return int(code.value)


def selftest_bounded_wait(limit_us, device_error, waited_ns=None, stream=None) -> None:
    """Run the kernels' bounded wait on a barrier nothing completes, for
    ``limit_us`` microseconds; it then sets DEVERR_TIMEOUT in ``device_error``
    and returns.  ``waited_ns``: optional int64 device tensor of one element,
    receives the waited time.  See include/pkv.h, pkv_selftest_bounded_wait."""
    lib = load_library()
    dv = device_error.device
    wn = _dev(waited_ns, "waited_ns", torch.int64, on=dv) if waited_ns is not None else None
    with _current(dv):
        st = lib.pkv_selftest_bounded_wait(int(limit_us),
                                           _dev(device_error, "device_error", torch.int32),
                                           wn, _stream_ptr(stream, dv))
    _raise(st, lib, "selftest_bounded_wait")


def version() -> int:
    return int(load_library().pkv_version())


def prefill_workspace_size(num_seqs, chunk_tokens, num_q_heads, num_kv_heads, head_dim,
                           max_blocks_per_seq, partition_tokens=0,
                           block_size=BLOCK_SIZE) -> int:
    """Bytes of workspace ``paged_attention_prefill`` needs (0: none)."""
    lib = load_library()
    return int(lib.pkv_prefill_workspace_size(num_seqs, chunk_tokens, num_q_heads, num_kv_heads,
                                              head_dim, max_blocks_per_seq, block_size,
                                              int(partition_tokens)))


def prefill_partition_tokens(num_seqs, chunk_tokens, num_q_heads, num_kv_heads, head_dim,
                             max_blocks_per_seq, block_size=BLOCK_SIZE) -> int:
    """Partition length a prefill call picks when ``partition_tokens`` is 0."""
    lib = load_library()
    return int(lib.pkv_prefill_partition_tokens(num_seqs, chunk_tokens, num_q_heads,
                                                num_kv_heads, head_dim, max_blocks_per_seq,
                                                block_size))


def paged_attention_prefill(q, k_cache, v_cache, block_tables, context_lens, scale, out,
                            stream=None, *, workspace=None, partition_tokens=0,
                            device_error=None, sliding_window=0) -> torch.Tensor:
    """Chunked prefill: the last C tokens of every sequence attend causally to
    its paged context (their K/V already appended), each to its last
    ``sliding_window`` tokens when that is > 0.  q [B, C, Hq, d] bf16,
    caches [NB, Hkv, 16, d] bf16, out [B, C, Hq, d] float32 or bfloat16;
    writes and returns ``out``.  See include/pkv.h, pkv_paged_attention_prefill.
    """
    lib = load_library()
    dv = q.device
    if q.dtype != torch.bfloat16 or k_cache.dtype != torch.bfloat16 \
            or v_cache.dtype != torch.bfloat16:
        raise TypeError("prefill: q and the caches must be bfloat16")
    B, C, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if v_cache.shape != k_cache.shape or d2 != d or out.shape != (B, C, Hq, d) \
            or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("inconsistent paged_attention_prefill shapes")
    need = lib.pkv_prefill_workspace_size(B, C, Hq, Hkv, d, MB, bs, int(partition_tokens))
    if workspace is None:
        workspace = torch.empty(max(int(need), 16), dtype=torch.uint8, device=q.device)
    err = (_dev(device_error, "device_error", torch.int32, on=dv)
           if device_error is not None else None)
    with _current(dv):
        st = lib.pkv_paged_attention_prefill(
            _dev(q, "q", on=dv), _dev(k_cache, "k_cache", on=dv), _dev(v_cache, "v_cache", on=dv),
            _dev(block_tables, "block_tables", torch.int32, on=dv),
            _dev(context_lens, "context_lens", torch.int32, on=dv), _dev(out, "out", on=dv),
            _dev(workspace, "workspace", on=dv), workspace.numel() * workspace.element_size(),
            B, C, Hq, Hkv, d, NB, bs, MB, PKV_DTYPE_BF16, _dtype_code(out.dtype), float(scale),
            int(sliding_window), int(partition_tokens), err, _stream_ptr(stream, q.device))
    _raise(st, lib, "paged_attention_prefill")
    return out


def decode_cascade_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                  max_blocks_per_seq, partition_tokens=0,
                                  block_size=BLOCK_SIZE) -> int:
    """Bytes of workspace ``paged_attention_decode_cascade`` needs."""
    lib = load_library()
    return int(lib.pkv_decode_cascade_workspace_size(num_seqs, num_q_heads, num_kv_heads,
                                                     head_dim, max_blocks_per_seq, block_size,
                                                     PKV_DTYPE_BF16, int(partition_tokens)))


def paged_attention_decode_cascade(q, k_cache, v_cache, block_tables, context_lens, group_start,
                                   shared_tokens, max_group_size, scale, out, stream=None, *,
                                   workspace=None, partition_tokens=0, force_simt=False,
                                   device_error=None, sliding_window=0) -> torch.Tensor:
    """``paged_attention_decode`` for groups of sequences that share prefix
    blocks: group g is sequences [group_start[g], group_start[g+1]) (int32,
    device), whose first shared_tokens[b] tokens (int32 [B], device) sit in
    the group's shared blocks.  Same result; each shared prefix is read once
    per group.  bf16 only; q already rotated.  ``sliding_window`` > 0: each
    query attends to the last ``sliding_window`` tokens of its context
    (pkv_paged_attention_decode_cascade_window).  See include/pkv.h."""
    lib = load_library()
    dv = q.device
    if q.dtype != torch.bfloat16 or k_cache.dtype != torch.bfloat16 \
            or v_cache.dtype != torch.bfloat16:
        raise TypeError("cascade: q and the caches must be bfloat16")
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    NG = max(0, group_start.numel() - 1)
    if v_cache.shape != k_cache.shape or d2 != d or out.shape != (B, Hq, d) \
            or block_tables.shape[0] != B or context_lens.shape != (B,) \
            or shared_tokens.shape != (B,):
        raise ValueError("inconsistent paged_attention_decode_cascade shapes")
    need = lib.pkv_decode_cascade_workspace_size(B, Hq, Hkv, d, MB, bs, PKV_DTYPE_BF16,
                                                 int(partition_tokens))
    if workspace is None:
        workspace = new_workspace(int(need), q.device)
    err = (_dev(device_error, "device_error", torch.int32, on=dv)
           if device_error is not None else None)
    head = (_dev(q, "q", on=dv), _dev(k_cache, "k_cache", on=dv),
            _dev(v_cache, "v_cache", on=dv),
            _dev(block_tables, "block_tables", torch.int32, on=dv),
            _dev(context_lens, "context_lens", torch.int32, on=dv),
            _dev(group_start, "group_start", torch.int32, on=dv) if NG else None,
            _dev(shared_tokens, "shared_tokens", torch.int32, on=dv), _dev(out, "out", on=dv),
            _dev(workspace, "workspace", on=dv), workspace.numel() * workspace.element_size(),
            B, NG, int(max_group_size), Hq, Hkv, d, NB, bs, MB, PKV_DTYPE_BF16,
            _dtype_code(out.dtype), float(scale))
    tail = (int(partition_tokens), _flags(force_simt, True), err, _stream_ptr(stream, q.device))
    with _current(dv):
        if sliding_window:
            st = lib.pkv_paged_attention_decode_cascade_window(*head, int(sliding_window), *tail)
        else:
            st = lib.pkv_paged_attention_decode_cascade(*head, *tail)
    _raise(st, lib, "paged_attention_decode_cascade")
    return out


def kv_request_bytes(num_layers, num_kv_heads, head_dim, tokens, kv_dtype=torch.bfloat16,
                     block_size=BLOCK_SIZE) -> int:
    """Cache bytes a request of ``tokens`` tokens occupies over ``num_layers``
    layers (whole blocks); see include/pkv.h, pkv_kv_request_bytes."""
    lib = load_library()
    n = int(lib.pkv_kv_request_bytes(num_layers, num_kv_heads, head_dim, block_size, tokens,
                                     _kv_dtype_code(kv_dtype)))
    if n < 0:
        raise ValueError("invalid KV accounting arguments")
    return n


def kv_admission_capacity(pool_bytes, num_layers, num_kv_heads, head_dim, tokens,
                          kv_dtype=torch.bfloat16, block_size=BLOCK_SIZE) -> int:
    """How many requests of ``tokens`` tokens fit in ``pool_bytes`` of cache."""
    lib = load_library()
    n = int(lib.pkv_kv_admission_capacity(int(pool_bytes), num_layers, num_kv_heads, head_dim,
                                          block_size, tokens, _kv_dtype_code(kv_dtype)))
    if n < 0:
        raise ValueError("invalid KV accounting arguments")
    return n


class BlockManager:
    """Host-side block allocator of a paged KV cache with prefix caching (the
    library's pkv_bm_* calls; see include/pkv.h).  Not thread safe."""

    def __init__(self, num_blocks: int, block_size: int = BLOCK_SIZE):
        self._lib = load_library()
        self._h = self._lib.pkv_bm_create(int(num_blocks), int(block_size))
        if not self._h:
            raise PkvError(1, f"pkv_bm_create: {self._lib.pkv_last_error().decode()}")
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)

    def close(self):
        if self._h:
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_sequence(self, seq_id: int, tokens) -> int:
        """Admit a sequence with its prompt token ids; returns how many of its
        leading tokens sit in reused (cached) blocks."""
        t = torch.as_tensor(tokens, dtype=torch.int32).contiguous()
        shared = ctypes.c_int32(0)
        _raise(self._lib.pkv_bm_add_sequence(self._h, int(seq_id), t.data_ptr() if t.numel() else None,
                                             t.numel(), ctypes.byref(shared)),
               self._lib, "pkv_bm_add_sequence")
        return int(shared.value)

    def prompt_slots(self, seq_id: int, num_tokens: int) -> torch.Tensor:
        """int64 [num_tokens] cache slot of each prompt token, -1 when reused."""
        out = torch.empty(int(num_tokens), dtype=torch.int64)
        _raise(self._lib.pkv_bm_prompt_slots(self._h, int(seq_id), out.data_ptr(), out.numel()),
               self._lib, "pkv_bm_prompt_slots")
        return out

    def append(self, seq_id: int, token: int) -> int:
        """Cache slot of the sequence's next token."""
        slot = ctypes.c_int64(0)
        _raise(self._lib.pkv_bm_append(self._h, int(seq_id), int(token), ctypes.byref(slot)),
               self._lib, "pkv_bm_append")
        return int(slot.value)

    def free_sequence(self, seq_id: int) -> None:
        _raise(self._lib.pkv_bm_free_sequence(self._h, int(seq_id)), self._lib,
               "pkv_bm_free_sequence")

    def block_table(self, seq_id: int, max_blocks: int) -> tuple[torch.Tensor, int]:
        """(int32 [max_blocks] table row padded with -1, number of tokens)."""
        row = torch.empty(int(max_blocks), dtype=torch.int32)
        nb, nt = ctypes.c_int32(0), ctypes.c_int64(0)
        _raise(self._lib.pkv_bm_block_table(self._h, int(seq_id), row.data_ptr(), row.numel(),
                                            ctypes.byref(nb), ctypes.byref(nt)),
               self._lib, "pkv_bm_block_table")
        return row, int(nt.value)

    def shared_tokens(self, seq_id: int) -> int:
        return int(self._lib.pkv_bm_shared_tokens(self._h, int(seq_id)))

    @property
    def free_blocks(self) -> int:
        return int(self._lib.pkv_bm_free_blocks(self._h))

    @property
    def cached_blocks(self) -> int:
        return int(self._lib.pkv_bm_cached_blocks(self._h))
