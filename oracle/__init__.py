"""fp64 CPU oracle for paged decode attention and the KV append.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library and its Python binding never do; the two share no
code.  The arithmetic lives in ``pkv_oracle.c`` (plain loops, fp64); this
module only marshals CPU tensors into it.

Functions (all take and return CPU ``torch`` tensors):

* ``kv_append``            -- RoPE on q (in place) and k, write k/v into the slot.
* ``paged_attention_decode`` -- plain two-pass softmax(q K^T scale) V over the
  tokens each block table lists, in fp64.
* ``paged_chunked_prefill`` -- a chunk of C queries per sequence, each a
  decode over its own causal prefix of the paged cache.
* ``contiguous_decode`` / ``causal_prefill`` -- the same definition without
  paging, used only to check the oracle itself.
* ``kv_append_e4m3`` / ``paged_attention_decode_e4m3`` -- the same append and
  decode over an 8-bit (E4M3 code x per-tensor scale) cache, whose V pages
  are stored transposed: k_cache [NB, Hkv, 16, d], v_cache [NB, Hkv, d, 16],
  both uint8.
* ``round_e4m3`` / ``e4m3_to_double`` -- the E4M3 rounding and decoding.
* ``rope`` / ``round_bf16`` / ``bf16_to_double`` -- the oracle's building blocks,
  exposed so that tests can pin them.
"""
from __future__ import annotations

import ctypes

import torch

from . import build as _build

F32, BF16, E4M3 = 0, 1, 2
_ERRORS = {
    -1: "invalid argument",
    -2: "block id out of range",
    -3: "context length out of range",
    -4: "slot out of range",
    -5: "out of memory",
}


class OracleError(RuntimeError):
    pass


class Oracle:
    """The oracle's functions bound to one build of ``pkv_oracle.c``.

    The default instance (module-level functions below) uses the library that
    ``oracle/build.py`` makes.  Tests may bind a separately compiled copy.
    """

    def __init__(self, path: str | None = None):
        self._path = path
        self._lib = None

    @property
    def lib(self):
        if self._lib is None:
            path = self._path or _build.build()
            lib = ctypes.CDLL(path)
            i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
            lib.orc_round_bf16.argtypes = [vp, vp, i64]
            lib.orc_bf16_to_double.argtypes = [vp, vp, i64]
            lib.orc_rope.argtypes = [vp, i64, i64, vp, dbl]
            lib.orc_kv_append.argtypes = [i32, vp, vp, vp, vp, vp, vp, vp,
                                          i64, i64, i64, i64, i64, i64, dbl]
            lib.orc_paged_decode.argtypes = [i32, i32, vp, vp, vp, vp, vp,
                                             i64, i64, i64, i64, i64, i64, i64, dbl, i64,
                                             vp, i64, i32, vp]
            lib.orc_paged_decode_e4m3.argtypes = [i32, vp, vp, vp, vp, vp,
                                                  i64, i64, i64, i64, i64, i64, i64, dbl, dbl,
                                                  dbl, i64, vp, i64, i32, vp]
            lib.orc_kv_append_e4m3.argtypes = [i32, vp, vp, vp, vp, vp, vp, vp,
                                               i64, i64, i64, i64, i64, i64, dbl, dbl, dbl]
            lib.orc_round_e4m3.argtypes = [vp, vp, i64]
            lib.orc_e4m3_to_double.argtypes = [vp, vp, i64]
            lib.orc_contiguous_decode.argtypes = [vp, vp, vp, i64, i64, i64, i64, dbl, vp]
            lib.orc_causal_prefill.argtypes = [vp, vp, vp, i64, i64, i64, i64, dbl, vp]
            for name in ("orc_round_bf16", "orc_bf16_to_double", "orc_rope", "orc_kv_append",
                         "orc_paged_decode", "orc_contiguous_decode", "orc_causal_prefill",
                         "orc_paged_decode_e4m3", "orc_kv_append_e4m3", "orc_round_e4m3",
                         "orc_e4m3_to_double"):
                getattr(lib, name).restype = ctypes.c_int
            self._lib = lib
        return self._lib

    def round_bf16(self, x: torch.Tensor) -> torch.Tensor:
        """Round float64 values to bf16 in one step (nearest, ties to even)."""
        x = _cpu(x.contiguous(), torch.float64)
        out = torch.empty(x.shape, dtype=torch.bfloat16)
        _check(self.lib.orc_round_bf16(_ptr(x), _ptr(out), x.numel()))
        return out

    def bf16_to_double(self, x: torch.Tensor) -> torch.Tensor:
        x = _cpu(x.contiguous(), torch.bfloat16)
        out = torch.empty(x.shape, dtype=torch.float64)
        _check(self.lib.orc_bf16_to_double(_ptr(x), _ptr(out), x.numel()))
        return out

    def round_e4m3(self, x: torch.Tensor) -> torch.Tensor:
        """uint8 E4M3 codes of float64 values: nearest, ties to even, saturating
        to +-448 (no binary32 step: that belongs to the cache quantizer)."""
        x = _cpu(x.contiguous(), torch.float64)
        out = torch.empty(x.shape, dtype=torch.uint8)
        _check(self.lib.orc_round_e4m3(_ptr(x), _ptr(out), x.numel()))
        return out

    def e4m3_to_double(self, c: torch.Tensor) -> torch.Tensor:
        c = _cpu(c.contiguous(), torch.uint8)
        out = torch.empty(c.shape, dtype=torch.float64)
        _check(self.lib.orc_e4m3_to_double(_ptr(c), _ptr(out), c.numel()))
        return out

    def rope(self, x: torch.Tensor, positions: torch.Tensor, theta: float) -> torch.Tensor:
        """Rotate-half RoPE in fp64.  x: [n, d] float64, positions: [n] int64."""
        x = _cpu(x, torch.float64).clone()
        positions = _cpu(positions.contiguous(), torch.int64)
        n, d = x.shape
        _check(self.lib.orc_rope(_ptr(x), n, d, _ptr(positions), float(theta)))
        return x

    def kv_append(self, q, k_new, v_new, positions, slot_mapping, k_cache, v_cache, rope_theta):
        """In-place: rotate q; write rotated k and unchanged v into the cache slots.

        q [T, Hq, d], k_new/v_new [T, Hkv, d], caches [NB, Hkv, bs, d]; one storage
        dtype (float32 or bfloat16) for all five; positions/slot_mapping int64 [T].
        """
        for t in (q, k_new, v_new, k_cache, v_cache):
            _cpu(t)
        dt = _storage_code(q)
        for t in (k_new, v_new, k_cache, v_cache):
            if t.dtype != q.dtype:
                raise TypeError("all append tensors share one dtype")
        _cpu(positions, torch.int64)
        _cpu(slot_mapping, torch.int64)
        T, Hq, d = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        _check(self.lib.orc_kv_append(dt, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(positions),
                                      _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache),
                                      T, Hq, Hkv, d, NB, bs, float(rope_theta)))

    def paged_attention_decode(self, q, k_cache, v_cache, block_tables, context_lens, scale,
                               pairs=None, nthreads: int = 1, window: int = 0) -> torch.Tensor:
        """fp64 [B, Hq, d] output of single-query attention over paged K/V.

        ``pairs`` ([n, 2] int64 of (b, h)) restricts the work to those outputs;
        the other rows of the result are left as NaN.  ``window`` > 0: each
        query attends to the last ``window`` tokens of its context only.
        """
        _cpu(q)
        _cpu(k_cache)
        _cpu(v_cache)
        _cpu(block_tables, torch.int32)
        _cpu(context_lens, torch.int32)
        if k_cache.dtype != v_cache.dtype:
            raise TypeError("k_cache and v_cache share one dtype")
        B, Hq, d = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
        out = torch.full((B, Hq, d), float("nan"), dtype=torch.float64)
        if pairs is not None:
            pairs = _cpu(pairs.contiguous(), torch.int64)
            pp, npairs = _ptr(pairs), pairs.shape[0]
        else:
            pp, npairs = None, 0
        _check(self.lib.orc_paged_decode(_storage_code(q), _storage_code(k_cache), _ptr(q),
                                         _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                         _ptr(context_lens), B, Hq, Hkv, d, NB, bs, MB,
                                         float(scale), int(window), pp, npairs, int(nthreads),
                                         _ptr(out)))
        return out

    def kv_append_e4m3(self, q, k_new, v_new, positions, slot_mapping, k_cache, v_cache,
                       rope_theta, k_scale, v_scale):
        """In-place: rotate q (its own dtype); write the E4M3 codes of rotated
        k / k_scale and of v / v_scale into the slots.  q, k_new, v_new share
        one dtype (float32 or bfloat16); k_cache [NB, Hkv, bs, d] and v_cache
        [NB, Hkv, d, bs] are uint8."""
        for t in (q, k_new, v_new, k_cache, v_cache):
            _cpu(t)
        dt = _storage_code(q)
        for t in (k_new, v_new):
            if t.dtype != q.dtype:
                raise TypeError("q, k_new and v_new share one dtype")
        for t in (k_cache, v_cache):
            if t.dtype != torch.uint8:
                raise TypeError("E4M3 caches are uint8")
        _cpu(positions, torch.int64)
        _cpu(slot_mapping, torch.int64)
        T, Hq, d = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        if v_cache.shape != (NB, Hkv, d, bs):
            raise ValueError("v_cache must be [NB, Hkv, d, bs]")
        _check(self.lib.orc_kv_append_e4m3(dt, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(positions),
                                           _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache),
                                           T, Hq, Hkv, d, NB, bs, float(rope_theta),
                                           float(k_scale), float(v_scale)))

    def paged_attention_decode_e4m3(self, q, k_cache, v_cache, block_tables, context_lens, scale,
                                    k_scale, v_scale, pairs=None, nthreads: int = 1,
                                    window: int = 0) -> torch.Tensor:
        """fp64 [B, Hq, d] decode over an E4M3 cache (k_cache [NB, Hkv, bs, d],
        v_cache [NB, Hkv, d, bs], uint8); ``pairs`` as in paged_attention_decode."""
        _cpu(q)
        _cpu(k_cache, torch.uint8)
        _cpu(v_cache, torch.uint8)
        _cpu(block_tables, torch.int32)
        _cpu(context_lens, torch.int32)
        B, Hq, d = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        if v_cache.shape != (NB, Hkv, d, bs):
            raise ValueError("v_cache must be [NB, Hkv, d, bs]")
        MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
        out = torch.full((B, Hq, d), float("nan"), dtype=torch.float64)
        if pairs is not None:
            pairs = _cpu(pairs.contiguous(), torch.int64)
            pp, npairs = _ptr(pairs), pairs.shape[0]
        else:
            pp, npairs = None, 0
        _check(self.lib.orc_paged_decode_e4m3(_storage_code(q), _ptr(q), _ptr(k_cache),
                                              _ptr(v_cache), _ptr(block_tables),
                                              _ptr(context_lens), B, Hq, Hkv, d, NB, bs, MB,
                                              float(scale), float(k_scale), float(v_scale),
                                              int(window), pp, npairs, int(nthreads), _ptr(out)))
        return out

    def paged_chunked_prefill(self, q, k_cache, v_cache, block_tables, context_lens, scale,
                              nthreads: int = 1, window: int = 0) -> torch.Tensor:
        """fp64 [B, C, Hq, d] output of a prefill chunk: the last C context
        tokens of each sequence, query i attending to tokens 0 .. L - C + i.

        "Efficient LLM Inference", KV Caching: Verify Reuse, Positions and
        Windows -- a chunk computed over the retained K/V equals the
        full-prefix pass, so query i of the chunk is exactly one decode step
        over the first L - C + i + 1 tokens.  That is how it is computed here:
        one plain decode per chunk position, with that context length (and
        the same sliding ``window``, when > 0).
        """
        _cpu(q)
        _cpu(context_lens, torch.int32)
        B, C, Hq, d = q.shape
        out = torch.empty((B, C, Hq, d), dtype=torch.float64)
        for i in range(C):
            lens_i = (context_lens.to(torch.int64) - C + i + 1).clamp(min=0).to(torch.int32)
            out[:, i] = self.paged_attention_decode(q[:, i].contiguous(), k_cache, v_cache,
                                                    block_tables, lens_i, scale,
                                                    nthreads=nthreads, window=window)
        return out

    def contiguous_decode(self, q, K, V, scale) -> torch.Tensor:
        """q [Hq, d], K/V [L, Hkv, d] (float64) -> [Hq, d]."""
        q, K, V = (_cpu(t.contiguous(), torch.float64) for t in (q, K, V))
        Hq, d = q.shape
        L, Hkv, _ = K.shape
        out = torch.empty((Hq, d), dtype=torch.float64)
        _check(self.lib.orc_contiguous_decode(_ptr(q), _ptr(K), _ptr(V), L, Hq, Hkv, d,
                                              float(scale), _ptr(out)))
        return out

    def causal_prefill(self, Q, K, V, scale) -> torch.Tensor:
        """Q [L, Hq, d], K/V [L, Hkv, d] (float64) -> [L, Hq, d], row r sees 0..r."""
        Q, K, V = (_cpu(t.contiguous(), torch.float64) for t in (Q, K, V))
        L, Hq, d = Q.shape
        Hkv = K.shape[1]
        out = torch.empty((L, Hq, d), dtype=torch.float64)
        _check(self.lib.orc_causal_prefill(_ptr(Q), _ptr(K), _ptr(V), L, Hq, Hkv, d,
                                           float(scale), _ptr(out)))
        return out


def _check(status: int) -> None:
    if status != 0:
        raise OracleError(_ERRORS.get(status, f"oracle error {status}"))


def _cpu(t: torch.Tensor, dtype=None) -> torch.Tensor:
    if t.device.type != "cpu":
        raise ValueError("the oracle takes CPU tensors")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("the oracle takes contiguous tensors")
    return t


def _storage_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported storage dtype {t.dtype}")


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr())


default = Oracle()
round_bf16 = default.round_bf16
bf16_to_double = default.bf16_to_double
rope = default.rope
kv_append = default.kv_append
paged_attention_decode = default.paged_attention_decode
contiguous_decode = default.contiguous_decode
causal_prefill = default.causal_prefill
paged_chunked_prefill = default.paged_chunked_prefill
round_e4m3 = default.round_e4m3
e4m3_to_double = default.e4m3_to_double
kv_append_e4m3 = default.kv_append_e4m3
paged_attention_decode_e4m3 = default.paged_attention_decode_e4m3
