"""The C-ABI library without a GPU: it loads, exports every symbol that
include/pkv.h declares, and rejects bad arguments on the host with the
documented status before any launch (no compute call is made here)."""
from __future__ import annotations

import ctypes
import math
import os
import re

import pytest

import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200 import build as lib_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
F32, BF16 = 0, 1


@pytest.fixture(scope="module")
def lib():
    lib_build.build()
    return pkv.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"pkv_kv_append", "pkv_paged_attention_decode", "pkv_decode_workspace_size"} <= set(names)
    for name in names:
        assert hasattr(lib, name), f"{name} declared in pkv.h but not exported"


def test_library_is_built_for_sm100a():
    log = os.path.join(lib_build.BUILD_DIR, "paged_decode.cu.log")
    assert os.path.exists(lib_build.LIB)
    assert "arch=compute_100a,code=sm_100a" in open(log).read()


def test_version_and_status_strings(lib):
    assert lib.pkv_version() >= 100
    assert lib.pkv_status_string(0) == b"ok"
    assert lib.pkv_status_string(3) == b"workspace too small"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation


def _append(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, pos=FAKE, slot=FAKE, kc=FAKE, vc=FAKE, T=1, Hq=8, Hkv=2, d=64,
             NB=4, bs=16, dtype=BF16, theta=1e4, err=None)
    a.update(kw)
    return lib.pkv_kv_append(a["q"], a["k"], a["v"], a["pos"], a["slot"], a["kc"], a["vc"], a["T"],
                             a["Hq"], a["Hkv"], a["d"], a["NB"], a["bs"], a["dtype"], a["theta"],
                             a["err"], None)


def _decode(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, out=FAKE, ws=None, wsb=0, B=2, Hq=8, Hkv=2,
             d=64, NB=4, bs=16, MB=4, kvdt=BF16, odt=BF16, scale=0.125, P=0, flags=0, err=None)
    a.update(kw)
    return lib.pkv_paged_attention_decode(a["q"], a["kc"], a["vc"], a["bt"], a["cl"], a["out"],
                                          a["ws"], a["wsb"], a["B"], a["Hq"], a["Hkv"], a["d"],
                                          a["NB"], a["bs"], a["MB"], a["kvdt"], a["odt"],
                                          a["scale"], a["P"], a["flags"], a["err"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(d=48), UNSUPPORTED),
    (dict(Hq=6, Hkv=2), UNSUPPORTED),     # group size 3
    (dict(Hq=7, Hkv=2), INVALID),         # not a multiple
    (dict(bs=32), UNSUPPORTED),
    (dict(dtype=7), UNSUPPORTED),
    (dict(theta=0.0), INVALID),
    (dict(T=-1), INVALID),
    (dict(q=None), INVALID),
    (dict(kc=FAKE + 8), INVALID),          # misaligned
    (dict(NB=0), INVALID),
    (dict(T=0, q=None, k=None), OK),       # empty: nothing to do, nothing launched
])
def test_kv_append_rejects_bad_arguments(lib, kw, status):
    assert _append(lib, **kw) == status
    if status != OK:
        assert lib.pkv_last_error() != b""


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), UNSUPPORTED),
    (dict(Hq=16, Hkv=1), UNSUPPORTED),     # group size 16
    (dict(bs=8), UNSUPPORTED),
    (dict(kvdt=2), UNSUPPORTED),
    (dict(odt=5), UNSUPPORTED),
    (dict(B=-1), INVALID),
    (dict(B=5000), UNSUPPORTED),           # over PKV_MAX_SEQS_PER_CALL
    (dict(flags=0x10), INVALID),
    (dict(scale=math.inf), INVALID),
    (dict(P=24), INVALID),                 # not a multiple of 16
    (dict(P=16, MB=2000), UNSUPPORTED),    # more than 1024 partitions
    (dict(out=None), INVALID),
    (dict(bt=FAKE + 2), INVALID),
    (dict(MB=0), INVALID),
    (dict(P=16, MB=4), WORKSPACE),         # split path needs a workspace
    (dict(P=16, MB=4, ws=FAKE, wsb=255), WORKSPACE),   # smaller than the plan
    (dict(P=16, MB=4, ws=FAKE + 4, wsb=1 << 20), WORKSPACE),   # misaligned
    (dict(B=0, q=None, out=None), OK),
])
def test_decode_rejects_bad_arguments(lib, kw, status):
    assert _decode(lib, **kw) == status



E4M3 = 2


def _append8(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, pos=FAKE, slot=FAKE, kv=FAKE, T=1, Hq=8, Hkv=2, d=64,
             NB=4, bs=16, dtype=BF16, theta=1e4, ks=0.05, vs=0.05, err=None)
    a.update(kw)
    return lib.pkv_kv_append_e4m3(a["q"], a["k"], a["v"], a["pos"], a["slot"], a["kv"],
                                  a["T"], a["Hq"], a["Hkv"], a["d"], a["NB"], a["bs"], a["dtype"],
                                  a["theta"], a["ks"], a["vs"], a["err"], None)


def _decode8(lib, **kw):
    a = dict(q=FAKE, kv=FAKE, bt=FAKE, cl=FAKE, out=FAKE, ws=None, wsb=0, B=2, Hq=8, Hkv=2,
             d=64, NB=4, bs=16, MB=4, odt=BF16, scale=0.125, ks=0.05, vs=0.05, P=0, flags=0,
             err=None)
    a.update(kw)
    return lib.pkv_paged_attention_decode_e4m3(
        a["q"], a["kv"], a["bt"], a["cl"], a["out"], a["ws"], a["wsb"], a["B"], a["Hq"],
        a["Hkv"], a["d"], a["NB"], a["bs"], a["MB"], a["odt"], a["scale"], a["ks"], a["vs"],
        a.get("win", 0), a["P"], a["flags"], a["err"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(ks=0.0), INVALID),
    (dict(vs=-1.0), INVALID),
    (dict(ks=math.inf), INVALID),
    (dict(vs=math.nan), INVALID),
    (dict(dtype=E4M3), UNSUPPORTED),       # q / k_new / v_new are float32 or bfloat16
    (dict(d=96), UNSUPPORTED),
    (dict(kv=FAKE + 8), INVALID),
    (dict(NB=1 << 26, Hkv=8, d=128), INVALID),   # byte rows past int32 tensor coordinates
    (dict(T=0, q=None, k=None), OK),
])
def test_kv_append_e4m3_rejects_bad_arguments(lib, kw, status):
    assert _append8(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(ks=0.0), INVALID),
    (dict(vs=math.nan), INVALID),
    (dict(flags=0x1), UNSUPPORTED),        # no CUDA-core kernel for the 8-bit cache
    (dict(odt=E4M3), UNSUPPORTED),
    (dict(d=96), UNSUPPORTED),
    (dict(P=16, MB=4), WORKSPACE),
    (dict(kv=FAKE + 4), INVALID),
    (dict(win=-1), INVALID),
    (dict(B=0, q=None, out=None), OK),
])
def test_decode_e4m3_rejects_bad_arguments(lib, kw, status):
    assert _decode8(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(win=-3), INVALID),
    (dict(win=16, kvdt=5), UNSUPPORTED),
    (dict(win=16, P=16, MB=4), WORKSPACE),
    (dict(win=16, B=0, q=None, out=None), OK),
])
def test_decode_window_rejects_bad_arguments(lib, kw, status):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, out=FAKE, ws=None, wsb=0, B=2, Hq=8, Hkv=2,
             d=64, NB=4, bs=16, MB=4, kvdt=BF16, odt=BF16, scale=0.125, P=0, flags=0, err=None)
    a.update(kw)
    st = lib.pkv_paged_attention_decode_window(
        a["q"], a["kc"], a["vc"], a["bt"], a["cl"], a["out"], a["ws"], a["wsb"], a["B"], a["Hq"],
        a["Hkv"], a["d"], a["NB"], a["bs"], a["MB"], a["kvdt"], a["odt"], a["scale"], a["win"],
        a["P"], a["flags"], a["err"], None)
    assert st == status


def test_e4m3_planning(lib):
    """The planning calls take the 8-bit cache dtype: the workspace follows
    the same formula; the CUDA-core kernel does not exist for it."""
    for P in (64, 1024):
        assert lib.pkv_decode_workspace_size(16, 32, 8, 128, 8193, 16, E4M3, P) == \
            lib.pkv_decode_workspace_size(16, 32, 8, 128, 8193, 16, BF16, P)
    # the automatic partition length depends on how many CTAs of the 8-bit
    # kernel fit on an SM; the workspace follows the same formula for it
    P8 = lib.pkv_decode_partition_tokens(16, 32, 8, 128, 8193, 16, E4M3)
    assert lib.pkv_decode_workspace_size(16, 32, 8, 128, 8193, 16, E4M3, 0) == \
        lib.pkv_decode_workspace_size(16, 32, 8, 128, 8193, 16, BF16, P8)
    assert lib.pkv_decode_partition_tokens(64, 32, 8, 64, 257, 16, E4M3) > 0
    assert lib.pkv_decode_launches(4, 32, 8, 64, 16, 16, E4M3, BF16, 0, 1, 0) == 0


def _step8(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, pos=FAKE, slot=FAKE, kv=FAKE, bt=FAKE, cl=FAKE, out=FAKE,
             ws=None, wsb=0, B=2, Hq=8, Hkv=2, d=64, NB=4, bs=16, MB=4, odt=BF16, theta=1e4,
             scale=0.125, ks=0.05, vs=0.05, win=0, P=0, flags=0, err=None)
    a.update(kw)
    return lib.pkv_decode_step_e4m3(
        a["q"], a["k"], a["v"], a["pos"], a["slot"], a["kv"], a["bt"], a["cl"], a["out"],
        a["ws"], a["wsb"], a["B"], a["Hq"], a["Hkv"], a["d"], a["NB"], a["bs"], a["MB"],
        a["odt"], a["theta"], a["scale"], a["ks"], a["vs"], a["win"], a["P"], a["flags"],
        a["err"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(ks=0.0), INVALID),
    (dict(vs=math.inf), INVALID),
    (dict(theta=0.0), INVALID),
    (dict(flags=0x1), UNSUPPORTED),        # no CUDA-core kernel for the 8-bit cache
    (dict(odt=E4M3), UNSUPPORTED),
    (dict(d=96), UNSUPPORTED),
    (dict(P=16, MB=4), WORKSPACE),
    (dict(kv=FAKE + 4), INVALID),
    (dict(k=FAKE + 8), INVALID),
    (dict(pos=FAKE + 4), INVALID),
    (dict(slot=None), INVALID),
    (dict(win=-1), INVALID),
    (dict(B=0, q=None, out=None), OK),
])
def test_decode_step_e4m3_rejects_bad_arguments(lib, kw, status):
    assert _step8(lib, **kw) == status

def test_workspace_size_formula(lib):
    # 16 sequences, 32/8 heads, d 128, contexts up to 8193 blocks, P = 1024
    n = lib.pkv_decode_workspace_size(16, 32, 8, 128, 8193, 16, BF16, 1024)
    NP = math.ceil(8193 * 16 / 1024)
    slots = 16 * 32 * NP
    a = lambda x: (x + 255) // 256 * 256
    # 256 bytes of scheduler counters, then the partial outputs and (m, l) pairs
    assert n == 256 + a(slots * 128 * 4) + a(slots * 2 * 4)
    # a single partition needs the counters only
    assert lib.pkv_decode_workspace_size(4, 8, 2, 64, 4, 16, BF16, 64) == 256
    assert lib.pkv_decode_workspace_size(4, 8, 2, 64, 4, 16, BF16, 24) == 0  # invalid P -> 0


def test_auto_partition_limits(lib):
    """Whole pages, at most 1024 partitions; batches that fill the GPU get
    whole 128-token stages.  (Without a device no cluster capacity is known,
    so small batches get the same rule here; the GPU tests check the
    cluster-mode choice.)"""
    for (B, MB) in ((1, 129), (64, 257), (256, 2049), (16, 8193), (4096, 3)):
        P = lib.pkv_decode_partition_tokens(B, 32, 8, 64, MB, 16, BF16)
        assert P % 16 == 0 and 16 <= P
        assert math.ceil(MB * 16 / P) <= 1024
    for (B, MB) in ((64, 257), (256, 2049), (16, 8193)):
        assert lib.pkv_decode_partition_tokens(B, 32, 8, 64, MB, 16, BF16) % 128 == 0


def test_prefill_workspace_size_formula(lib):
    # 4 sequences, chunk 8, 32/8 heads, d 64, contexts up to 129 blocks, P = 256
    n = lib.pkv_prefill_workspace_size(4, 8, 32, 8, 64, 129, 16, 256)
    NP = math.ceil(129 * 16 / 256)
    slots = 4 * 8 * 32 * NP
    a = lambda x: (x + 255) // 256 * 256
    assert n == a(slots * 64 * 4) + a(slots * 2 * 4)
    assert lib.pkv_prefill_workspace_size(4, 8, 32, 8, 64, 16, 16, 256) == 0   # one partition
    assert lib.pkv_prefill_workspace_size(4, 0, 32, 8, 64, 16, 16, 256) == 0   # no chunk


def _prefill(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, out=FAKE, ws=None, wsb=0, B=2, C=4,
             Hq=8, Hkv=2, d=64, NB=4, bs=16, MB=4, kvdt=BF16, odt=BF16, scale=0.125, P=0,
             err=None)
    a.update(kw)
    return lib.pkv_paged_attention_prefill(a["q"], a["kc"], a["vc"], a["bt"], a["cl"], a["out"],
                                           a["ws"], a["wsb"], a["B"], a["C"], a["Hq"], a["Hkv"],
                                           a["d"], a["NB"], a["bs"], a["MB"], a["kvdt"],
                                           a["odt"], a["scale"], a.get("win", 0), a["P"],
                                           a["err"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(win=-1), INVALID),
    (dict(kvdt=F32), UNSUPPORTED),          # bf16 only
    (dict(C=0), INVALID),
    (dict(C=65), INVALID),                  # longer than max_blocks * 16
    (dict(d=96), UNSUPPORTED),
    (dict(P=24), INVALID),
    (dict(q=None), INVALID),
    (dict(P=16, MB=4), WORKSPACE),          # split: needs a workspace
    (dict(B=0, q=None, out=None), OK),
])
def test_prefill_rejects_bad_arguments(lib, kw, status):
    assert _prefill(lib, **kw) == status


def _step(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, pos=FAKE, slot=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE,
             out=FAKE, ws=None, wsb=0, B=2, Hq=8, Hkv=2, d=64, NB=4, bs=16, MB=4, kvdt=BF16,
             odt=BF16, theta=1e4, scale=0.125, P=0, flags=0, err=None)
    a.update(kw)
    return lib.pkv_decode_step(a["q"], a["k"], a["v"], a["pos"], a["slot"], a["kc"], a["vc"],
                               a["bt"], a["cl"], a["out"], a["ws"], a["wsb"], a["B"], a["Hq"],
                               a["Hkv"], a["d"], a["NB"], a["bs"], a["MB"], a["kvdt"], a["odt"],
                               a["theta"], a["scale"], a["P"], a["flags"], a["err"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(theta=0.0), INVALID),
    (dict(theta=math.nan), INVALID),
    (dict(kvdt=E4M3), UNSUPPORTED),        # the 8-bit cache has no fused step
    (dict(d=96), UNSUPPORTED),
    (dict(Hq=24, Hkv=2), UNSUPPORTED),     # group size 12
    (dict(flags=0x10), INVALID),
    (dict(scale=-math.inf), INVALID),
    (dict(k=None), INVALID),
    (dict(slot=None), INVALID),
    (dict(v=FAKE + 8), INVALID),           # new rows 16-byte aligned
    (dict(pos=FAKE + 4), INVALID),         # int64 arrays 8-byte aligned
    (dict(P=16, MB=4), WORKSPACE),         # split path needs a workspace
    (dict(P=16, MB=4, ws=FAKE, wsb=64), WORKSPACE),
    (dict(B=0, q=None, k=None, out=None), OK),
])
def test_decode_step_rejects_bad_arguments(lib, kw, status):
    assert _step(lib, **kw) == status
    if status != OK:
        assert lib.pkv_last_error() != b""


def _cascade(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, gs=FAKE, sh=FAKE, out=FAKE, ws=None,
             wsb=0, B=8, G=1, MG=8, Hq=8, Hkv=2, d=64, NB=64, bs=16, MB=8, kvdt=BF16, odt=BF16,
             scale=0.125, P=0, flags=0, err=None)
    a.update(kw)
    return lib.pkv_paged_attention_decode_cascade(
        a["q"], a["kc"], a["vc"], a["bt"], a["cl"], a["gs"], a["sh"], a["out"], a["ws"], a["wsb"],
        a["B"], a["G"], a["MG"], a["Hq"], a["Hkv"], a["d"], a["NB"], a["bs"], a["MB"], a["kvdt"],
        a["odt"], a["scale"], a["P"], a["flags"], a["err"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(kvdt=F32), UNSUPPORTED),         # bf16 cache only
    (dict(odt=E4M3), UNSUPPORTED),
    (dict(d=80), UNSUPPORTED),
    (dict(B=257, MG=8), UNSUPPORTED),      # over 256 sequences
    (dict(flags=0x2), INVALID),            # only the CUDA-core flag applies
    (dict(G=-1), INVALID),
    (dict(MG=0), INVALID),                 # a group needs a member
    (dict(MG=9), INVALID),                 # larger than the batch
    (dict(scale=math.nan), INVALID),
    (dict(NB=0), INVALID),
    (dict(sh=None), INVALID),
    (dict(gs=None), INVALID),              # groups given, no offsets
    (dict(gs=FAKE + 2), INVALID),
    (dict(MB=0), INVALID),
    (dict(gs=None, G=0), WORKSPACE),       # no groups: only the workspace is missing
    (dict(ws=FAKE, wsb=255), WORKSPACE),
    (dict(B=0, G=0, q=None, out=None), OK),
])
def test_cascade_rejects_bad_arguments(lib, kw, status):
    assert _cascade(lib, **kw) == status
    if status != OK:
        assert lib.pkv_last_error() != b""


@pytest.mark.parametrize("kw,status", [
    (dict(win=-1), INVALID),
    (dict(win=64, kvdt=F32), UNSUPPORTED),
    (dict(win=64, MG=9), INVALID),
    (dict(win=64, ws=FAKE, wsb=255), WORKSPACE),
    (dict(win=64, B=0, G=0, q=None, out=None), OK),
])
def test_cascade_window_rejects_bad_arguments(lib, kw, status):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, gs=FAKE, sh=FAKE, out=FAKE, ws=None,
             wsb=0, B=8, G=1, MG=8, Hq=8, Hkv=2, d=64, NB=64, bs=16, MB=8, kvdt=BF16, odt=BF16,
             scale=0.125, win=0, P=0, flags=0, err=None)
    a.update(kw)
    st = lib.pkv_paged_attention_decode_cascade_window(
        a["q"], a["kc"], a["vc"], a["bt"], a["cl"], a["gs"], a["sh"], a["out"], a["ws"], a["wsb"],
        a["B"], a["G"], a["MG"], a["Hq"], a["Hkv"], a["d"], a["NB"], a["bs"], a["MB"], a["kvdt"],
        a["odt"], a["scale"], a["win"], a["P"], a["flags"], a["err"], None)
    assert st == status


def test_cascade_workspace_size_formula(lib):
    """256 bytes of scheduler counters, then NP + 1 partial slots per
    (sequence, q head): slot 0 holds the shared-prefix pass."""
    a = lambda x: (x + 255) // 256 * 256
    B, Hq, d, MB, P = 64, 32, 64, 2049, 512
    NP = math.ceil(MB * 16 / P)
    slots = B * Hq * (NP + 1)
    assert lib.pkv_decode_cascade_workspace_size(B, Hq, 8, d, MB, 16, BF16, P) == \
        256 + a(slots * d * 4) + a(slots * 2 * 4)
    # one partition still keeps the prefix slot
    slots = 4 * 8 * 2
    assert lib.pkv_decode_cascade_workspace_size(4, 8, 2, 64, 4, 16, BF16, 64) == \
        256 + a(slots * 64 * 4) + a(slots * 2 * 4)
    assert lib.pkv_decode_cascade_workspace_size(4, 8, 2, 64, 4, 16, F32, 64) == 0    # bf16 only
    assert lib.pkv_decode_cascade_workspace_size(4, 8, 2, 64, 4, 16, BF16, 24) == 0   # bad P
    assert lib.pkv_decode_cascade_workspace_size(-1, 8, 2, 64, 4, 16, BF16, 64) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), UNSUPPORTED),             # invalid shapes need no scratch: plain checks
    (dict(kvdt=7), UNSUPPORTED),
    # 64 x 32 heads x 64 partitions of d=128 partials: more than the 16 MiB scratch
    (dict(B=64, Hq=32, Hkv=8, d=128, MB=512, P=128), WORKSPACE),
])
def test_noalloc_rejects_before_touching_the_device(lib, kw, status):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, out=FAKE, B=2, Hq=8, Hkv=2, d=64, NB=4,
             bs=16, MB=4, kvdt=BF16, odt=BF16, scale=0.125, P=0, flags=0, err=None)
    a.update(kw)
    st = lib.pkv_paged_attention_decode_noalloc(
        a["q"], a["kc"], a["vc"], a["bt"], a["cl"], a["out"], a["B"], a["Hq"], a["Hkv"], a["d"],
        a["NB"], a["bs"], a["MB"], a["kvdt"], a["odt"], a["scale"], a["P"], a["flags"], a["err"],
        None)
    assert st == status


def test_device_error_reader_and_wait_selftest_reject_bad_arguments(lib):
    """Both diagnostics refuse their bad arguments on the host (no copy, no
    launch): null pointers, and a self-test limit outside 1 us .. 2 s."""
    code = ctypes.c_int32(7)
    assert lib.pkv_get_device_error(None, None, ctypes.byref(code)) == INVALID
    assert lib.pkv_get_device_error(FAKE, None, None) == INVALID
    assert code.value == 7
    assert lib.pkv_selftest_bounded_wait(0, FAKE, None, None) == INVALID
    assert lib.pkv_selftest_bounded_wait(2_000_001, FAKE, None, None) == INVALID
    assert lib.pkv_selftest_bounded_wait(1000, None, None, None) == INVALID
    assert lib.pkv_status_string(5) == b"device error word set by a kernel"
