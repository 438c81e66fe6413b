"""The Python binding's argument marshalling, without a GPU.

Every tensor argument reaches the C ABI as its device address, in the order
include/pkv.h declares, after the binding checks that it is a contiguous CUDA
tensor of the right dtype on the call's device (that of q): a kernel must
never be handed another GPU's memory.  Here the tensors are CPU tensors that
report themselves as CUDA tensors on a chosen device, and the library is a
recorder that returns "ok"; nothing is launched.
"""
from __future__ import annotations

import pytest
import torch

from paged_kv_cache_484_b200 import _binding as B

bf16, f32, i32, i64, u8 = torch.bfloat16, torch.float32, torch.int32, torch.int64, torch.uint8


class FakeCuda(torch.Tensor):
    """A CPU tensor that says it lives on cuda:<index>."""

    @staticmethod
    def of(t: torch.Tensor, index: int = 0) -> "FakeCuda":
        f = torch.Tensor._make_subclass(FakeCuda, t)
        f._fake_index = index
        return f

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return torch.device("cuda", self._fake_index)


class Recorder:
    """Stands in for the loaded library: every entry point returns 0 and
    records its arguments."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("pkv_"):
            raise AttributeError(name)

        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(B, "load_library", lambda: r)
    monkeypatch.setattr(B, "_stream_ptr", lambda stream, device: 0)
    return r


def _t(shape, dtype, index=0):
    return FakeCuda.of(torch.zeros(shape, dtype=dtype), index)


Bs, Hq, Hkv, D, NB, MB, C = 2, 8, 2, 64, 6, 3, 4


def _decode_args(dtype=bf16):
    return dict(q=_t((Bs, Hq, D), dtype), k_cache=_t((NB, Hkv, 16, D), dtype),
                v_cache=_t((NB, Hkv, 16, D), dtype), block_tables=_t((Bs, MB), i32),
                context_lens=_t((Bs,), i32), out=_t((Bs, Hq, D), f32))


def _step_args():
    a = _decode_args()
    a.update(k_new=_t((Bs, Hkv, D), bf16), v_new=_t((Bs, Hkv, D), bf16),
             positions=_t((Bs,), i64), slot_mapping=_t((Bs,), i64))
    return a


# (name, the call, its tensors by name, the C entry point, the tensors in ABI order)
def _cases():
    ws = lambda: _t((4096,), u8)
    err = lambda: _t((1,), i32)
    cases = []

    a = dict(_step_args(), err=err())
    cases.append(("kv_append", lambda a=a: B.kv_append(
        a["q"], a["k_new"], a["v_new"], a["positions"], a["slot_mapping"], a["k_cache"],
        a["v_cache"], 1e4, device_error=a["err"]), a, "pkv_kv_append",
        ["q", "k_new", "v_new", "positions", "slot_mapping", "k_cache", "v_cache"]))

    a = dict(_decode_args(), workspace=ws(), err=err())
    cases.append(("paged_attention_decode", lambda a=a: B.paged_attention_decode(
        a["q"], a["k_cache"], a["v_cache"], a["block_tables"], a["context_lens"], 0.125, a["out"],
        workspace=a["workspace"], device_error=a["err"]), a, "pkv_paged_attention_decode",
        ["q", "k_cache", "v_cache", "block_tables", "context_lens", "out", "workspace"]))

    a = dict(_decode_args(), workspace=ws(), err=err())
    cases.append(("paged_attention_decode window", lambda a=a: B.paged_attention_decode(
        a["q"], a["k_cache"], a["v_cache"], a["block_tables"], a["context_lens"], 0.125, a["out"],
        workspace=a["workspace"], device_error=a["err"], sliding_window=32), a,
        "pkv_paged_attention_decode_window",
        ["q", "k_cache", "v_cache", "block_tables", "context_lens", "out", "workspace"]))

    a = dict(_step_args(), workspace=ws(), err=err())
    cases.append(("decode_step", lambda a=a: B.decode_step(
        a["q"], a["k_new"], a["v_new"], a["positions"], a["slot_mapping"], a["k_cache"],
        a["v_cache"], a["block_tables"], a["context_lens"], 1e4, 0.125, a["out"],
        workspace=a["workspace"], device_error=a["err"]), a, "pkv_decode_step",
        ["q", "k_new", "v_new", "positions", "slot_mapping", "k_cache", "v_cache",
         "block_tables", "context_lens", "out", "workspace"]))

    a = dict(_step_args(), workspace=ws(), err=err())
    cases.append(("decode_step window", lambda a=a: B.decode_step(
        a["q"], a["k_new"], a["v_new"], a["positions"], a["slot_mapping"], a["k_cache"],
        a["v_cache"], a["block_tables"], a["context_lens"], 1e4, 0.125, a["out"],
        workspace=a["workspace"], device_error=a["err"], sliding_window=32), a,
        "pkv_decode_step_window",
        ["q", "k_new", "v_new", "positions", "slot_mapping", "k_cache", "v_cache",
         "block_tables", "context_lens", "out", "workspace"]))

    a = dict(_decode_args(), err=err())
    cases.append(("paged_attention_decode_noalloc", lambda a=a: B.paged_attention_decode_noalloc(
        a["q"], a["k_cache"], a["v_cache"], a["block_tables"], a["context_lens"], 0.125, a["out"],
        device_error=a["err"]), a, "pkv_paged_attention_decode_noalloc",
        ["q", "k_cache", "v_cache", "block_tables", "context_lens", "out"]))

    a = dict(_step_args(), kv_cache=_t((NB, Hkv, 2, 16 * D), u8), err=err())
    cases.append(("kv_append_e4m3", lambda a=a: B.kv_append_e4m3(
        a["q"], a["k_new"], a["v_new"], a["positions"], a["slot_mapping"], a["kv_cache"],
        1e4, 0.05, 0.05, device_error=a["err"]), a, "pkv_kv_append_e4m3",
        ["q", "k_new", "v_new", "positions", "slot_mapping", "kv_cache"]))

    a = dict(_decode_args(), kv_cache=_t((NB, Hkv, 2, 16 * D), u8), workspace=ws(), err=err())
    cases.append(("paged_attention_decode_e4m3", lambda a=a: B.paged_attention_decode_e4m3(
        a["q"], a["kv_cache"], a["block_tables"], a["context_lens"], 0.125, 0.05,
        0.05, a["out"], workspace=a["workspace"], device_error=a["err"]), a,
        "pkv_paged_attention_decode_e4m3",
        ["q", "kv_cache", "block_tables", "context_lens", "out", "workspace"]))

    a = dict(_step_args(), kv_cache=_t((NB, Hkv, 2, 16 * D), u8), workspace=ws(), err=err())
    cases.append(("decode_step_e4m3", lambda a=a: B.decode_step_e4m3(
        a["q"], a["k_new"], a["v_new"], a["positions"], a["slot_mapping"], a["kv_cache"],
        a["block_tables"], a["context_lens"], 1e4, 0.125, 0.05, 0.05, a["out"],
        workspace=a["workspace"], device_error=a["err"], sliding_window=48), a,
        "pkv_decode_step_e4m3",
        ["q", "k_new", "v_new", "positions", "slot_mapping", "kv_cache", "block_tables",
         "context_lens", "out", "workspace"]))

    a = dict(_decode_args(), q=_t((Bs, C, Hq, D), bf16), out=_t((Bs, C, Hq, D), f32),
             workspace=ws(), err=err())
    cases.append(("paged_attention_prefill", lambda a=a: B.paged_attention_prefill(
        a["q"], a["k_cache"], a["v_cache"], a["block_tables"], a["context_lens"], 0.125, a["out"],
        workspace=a["workspace"], device_error=a["err"]), a, "pkv_paged_attention_prefill",
        ["q", "k_cache", "v_cache", "block_tables", "context_lens", "out", "workspace"]))

    a = dict(_decode_args(), group_start=_t((2,), i32), shared_tokens=_t((Bs,), i32),
             workspace=ws(), err=err())
    cases.append(("paged_attention_decode_cascade", lambda a=a: B.paged_attention_decode_cascade(
        a["q"], a["k_cache"], a["v_cache"], a["block_tables"], a["context_lens"],
        a["group_start"], a["shared_tokens"], 2, 0.125, a["out"], workspace=a["workspace"],
        device_error=a["err"]), a, "pkv_paged_attention_decode_cascade",
        ["q", "k_cache", "v_cache", "block_tables", "context_lens", "group_start",
         "shared_tokens", "out", "workspace"]))

    a = dict(_decode_args(), group_start=_t((2,), i32), shared_tokens=_t((Bs,), i32),
             workspace=ws(), err=err())
    cases.append(("paged_attention_decode_cascade window",
                  lambda a=a: B.paged_attention_decode_cascade(
                      a["q"], a["k_cache"], a["v_cache"], a["block_tables"], a["context_lens"],
                      a["group_start"], a["shared_tokens"], 2, 0.125, a["out"],
                      workspace=a["workspace"], device_error=a["err"], sliding_window=64), a,
                  "pkv_paged_attention_decode_cascade_window",
                  ["q", "k_cache", "v_cache", "block_tables", "context_lens", "group_start",
                   "shared_tokens", "out", "workspace"]))
    return cases


CASES = _cases()


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tensors_reach_the_abi_as_addresses_in_declared_order(rec, case):
    _, call, tensors, entry, order = case
    call()
    assert [c[0] for c in rec.calls if not c[0].endswith("_size")] == [entry]
    args = [c for c in rec.calls if c[0] == entry][0][1]
    want = [tensors[n].data_ptr() for n in order]
    assert list(args[:len(order)]) == want
    # the device error word is passed too, after the sizes and before the stream
    assert tensors["err"].data_ptr() in args[len(order):]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_a_tensor_on_another_gpu_is_refused_before_the_call(rec, case):
    name, call, tensors, entry, order = case
    for moved in [n for n in order if n != "q"] + ["err"]:
        tensors[moved]._fake_index = 1
        label = "device_error" if moved == "err" else moved
        with pytest.raises(ValueError, match=f"{label} is on cuda:1"):
            call()
        tensors[moved]._fake_index = 0
    assert all(c[0] != entry for c in rec.calls)


def test_prepared_step_checks_devices_once(rec):
    a = dict(_step_args(), workspace=_t((4096,), u8))
    a["out"]._fake_index = 1
    with pytest.raises(ValueError, match="out is on cuda:1"):
        B.prepare_decode_step(a["q"], a["k_new"], a["v_new"], a["positions"],
                              a["slot_mapping"], a["k_cache"], a["v_cache"], a["block_tables"],
                              a["context_lens"], 1e4, 0.125, a["out"], workspace=a["workspace"])


def test_fused_window_step_passes_the_window_before_the_partition_length(rec):
    a = dict(_step_args(), workspace=_t((4096,), u8))
    B.decode_step(a["q"], a["k_new"], a["v_new"], a["positions"], a["slot_mapping"],
                  a["k_cache"], a["v_cache"], a["block_tables"], a["context_lens"], 1e4, 0.125,
                  a["out"], workspace=a["workspace"], partition_tokens=48, sliding_window=33)
    args = [c for c in rec.calls if c[0] == "pkv_decode_step_window"][0][1]
    # ..., rope_theta, scale, sliding_window, partition_tokens, flags, device_error, stream
    assert args[-7:-3] == (1e4, 0.125, 33, 48)


def test_e4m3_step_passes_scales_and_window_in_declared_order(rec):
    a = dict(_step_args(), kv_cache=_t((NB, Hkv, 2, 16 * D), u8), workspace=_t((4096,), u8))
    B.decode_step_e4m3(a["q"], a["k_new"], a["v_new"], a["positions"], a["slot_mapping"],
                       a["kv_cache"], a["block_tables"], a["context_lens"], 5e5, 0.125, 0.25,
                       0.5, a["out"], workspace=a["workspace"], sliding_window=48,
                       partition_tokens=64)
    (name, args), = rec.calls
    assert name == "pkv_decode_step_e4m3"
    # ... out, workspace, bytes, B, Hq, Hkv, d, NB, bs, MB, out_dtype, theta, scale,
    # k_scale, v_scale, window, P, flags, device_error, stream
    assert list(args[10:]) == [4096, Bs, Hq, Hkv, D, NB, 16, MB, 0, 5e5, 0.125, 0.25, 0.5, 48,
                               64, 0, None, 0]
