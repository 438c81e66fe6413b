"""The kernels' own checks of device-resident values, on the GPU.

The library never reads block tables, context lengths or slots on the host;
the kernels range-check every such value before using it.  A bad value sets
a PKV_DEVERR_* bit in the caller's error word and the access it would have
made is skipped.  These tests hand each kernel block-table entries of -7 and
num_blocks + 5, and context lengths past the table or below zero, and check:

* the right bit is set, and pkv_get_device_error reports it;
* every output is finite, and the sequences without a bad value still match
  the fp64 oracle (run on host copies of the pristine inputs);
* no cache row outside the step's own slots changed.

None of these inputs can fault: every bad value is rejected before the copy
or load it would address is issued.  The last test runs the bounded in-kernel
wait on a barrier nothing completes, with a short limit, and checks that it
gives up with PKV_DEVERR_TIMEOUT and returns.
"""
from __future__ import annotations

import pytest
import torch

import oracle
import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200 import workloads as W
from tests.parity_util import TOL_BF16, SubProblem

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LENS = [300, 700, 129, 1000]
GOOD, BAD = [0, 2], [1, 3]


def _workload(d=64, G=4, seed=71):
    return W.build_workload("devcheck", LENS, G * 2, 2, d, torch.bfloat16, 5e5, seed=seed,
                            device=DEV, pool_factor=1.3)


def _corrupt_tables(w):
    """-7 in sequence 1's sixth block, num_blocks + 5 in sequence 3's 21st."""
    t = w.block_tables.clone()
    t[1, 5] = -7
    t[3, 20] = w.num_blocks + 5
    return t


def _err():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def _oracle_decode(sub, seqs_out):
    out = oracle.paged_attention_decode(sub.q, sub.k_cache, sub.v_cache, sub.tables,
                                        sub.decode_lens, sub.scale, nthreads=8)
    return out


def _close(got, want, what):
    got = got.double().cpu()
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    err = (got - want).abs().max().item()
    assert err <= TOL_BF16, f"{what}: max err {err:.3e}"


@pytest.mark.parametrize("simt", [False, True])
@pytest.mark.parametrize("P", [0, 64])
def test_decode_bad_block_ids(simt, P):
    w = _workload()
    sub = SubProblem(w, GOOD)
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    tables = _corrupt_tables(w)
    err = _err()
    out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device=DEV)
    pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, tables, w.cached_lens, w.scale, out,
                               partition_tokens=P, force_simt=simt, device_error=err)
    code = pkv.get_device_error(err)
    assert code == pkv.DEVERR_BLOCK_ID
    assert torch.isfinite(out).all()
    assert torch.equal(w.k_cache, k0) and torch.equal(w.v_cache, v0)
    sub.decode_lens = sub.decode_lens - 1          # this call decodes the cached tokens only
    _close(out[GOOD], _oracle_decode(sub, GOOD), f"decode simt={simt} P={P}")


@pytest.mark.parametrize("P", [0, 128])
def test_decode_step_bad_block_ids(P):
    """The fused step still appends every sequence whose slot matches its
    table, and writes nothing else."""
    w = _workload()
    sub = SubProblem(w, GOOD)
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    tables = _corrupt_tables(w)
    err = _err()
    out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device=DEV)
    pkv.decode_step(w.q, w.k_new, w.v_new, w.positions, w.slot_mapping, w.k_cache, w.v_cache,
                    tables, w.decode_lens, w.rope_theta, w.scale, out, partition_tokens=P,
                    device_error=err)
    assert pkv.get_device_error(err) == pkv.DEVERR_BLOCK_ID
    assert torch.isfinite(out).all()
    # only the four appended rows differ
    slots = w.slot_mapping.cpu().tolist()
    changed = (w.k_cache != k0).any(dim=-1) | (w.v_cache != v0).any(dim=-1)   # [NB, Hkv, 16]
    rows = {(int(b), int(r)) for b, h, r in changed.nonzero().cpu().tolist()}
    assert rows <= {(s // 16, s % 16) for s in slots}
    _close(out[GOOD], sub.oracle_step(nthreads=8)[3], f"decode_step P={P}")


def test_decode_bad_context_lengths():
    """A length past the table's reach is flagged and clamped (the padding
    entries it then meets are flagged too); a negative one gives a zero row."""
    w = _workload(d=128, G=2, seed=73)
    sub = SubProblem(w, GOOD)
    lens = w.cached_lens.clone()
    lens[1] = w.max_blocks * 16 + 5
    lens[3] = -3
    err = _err()
    out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device=DEV)
    pkv.paged_attention_decode(w.q, w.k_cache, w.v_cache, w.block_tables, lens, w.scale, out,
                               partition_tokens=128, device_error=err)
    code = pkv.get_device_error(err)
    assert code & pkv.DEVERR_CONTEXT_LEN
    assert code & ~(pkv.DEVERR_CONTEXT_LEN | pkv.DEVERR_BLOCK_ID) == 0
    assert torch.isfinite(out).all()
    assert not out[3].any()
    sub.decode_lens = sub.decode_lens - 1
    _close(out[GOOD], _oracle_decode(sub, GOOD), "decode, bad lengths")


def test_decode_e4m3_bad_block_ids():
    w = _workload(seed=75)
    k8, v8, ks, vs = W.e4m3_cache(w)
    pristine = dict(q=w.q.cpu(), k=k8.cpu(), v=v8.cpu(), t=w.block_tables.cpu(),
                    l=w.cached_lens.cpu())
    tables = _corrupt_tables(w)
    err = _err()
    out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device=DEV)
    kv8 = W.e4m3_pack(k8, v8)
    pkv.paged_attention_decode_e4m3(w.q, kv8, tables, w.cached_lens, w.scale, ks, vs, out,
                                    partition_tokens=64, device_error=err)
    assert pkv.get_device_error(err) == pkv.DEVERR_BLOCK_ID
    assert torch.isfinite(out).all()
    assert torch.equal(kv8.cpu(), W.e4m3_pack(pristine["k"], pristine["v"]))
    want = oracle.paged_attention_decode_e4m3(pristine["q"], pristine["k"], pristine["v"],
                                              pristine["t"], pristine["l"], w.scale, ks, vs,
                                              nthreads=8)
    _close(out[GOOD], want[GOOD], "e4m3 decode")


def test_prefill_bad_block_ids_and_lengths():
    w = _workload(seed=77)
    C = 8
    g = torch.Generator(device=DEV)
    g.manual_seed(78)
    q = torch.randn((w.B, C, w.Hq, w.d), generator=g, device=DEV, dtype=torch.bfloat16)
    pristine = dict(q=q.cpu(), k=w.k_cache.cpu(), v=w.v_cache.cpu(), t=w.block_tables.cpu(),
                    l=w.cached_lens.cpu())
    tables = _corrupt_tables(w)
    err = _err()
    out = torch.full((w.B, C, w.Hq, w.d), float("nan"), dtype=torch.float32, device=DEV)
    pkv.paged_attention_prefill(q, w.k_cache, w.v_cache, tables, w.cached_lens, w.scale, out,
                                partition_tokens=128, device_error=err)
    assert pkv.get_device_error(err) == pkv.DEVERR_BLOCK_ID
    assert torch.isfinite(out).all()
    want = oracle.paged_chunked_prefill(pristine["q"], pristine["k"], pristine["v"],
                                        pristine["t"], pristine["l"], w.scale, nthreads=8)
    _close(out[GOOD], want[GOOD], "prefill, bad ids")
    # a context past the table's reach: flagged and clamped, output finite
    lens = w.cached_lens.clone()
    lens[2] = w.max_blocks * 16 + 9
    err.zero_()
    pkv.paged_attention_prefill(q, w.k_cache, w.v_cache, w.block_tables, lens, w.scale, out,
                                partition_tokens=128, device_error=err)
    assert pkv.get_device_error(err) & pkv.DEVERR_CONTEXT_LEN
    assert torch.isfinite(out).all()
    assert torch.equal(w.k_cache.cpu(), pristine["k"])


def test_bounded_wait_gives_up_and_returns():
    """The wait every pipeline stage uses, on a barrier nothing completes:
    after its limit it sets PKV_DEVERR_TIMEOUT and the kernel returns; the
    context stays usable for the next launch."""
    err = _err()
    waited = torch.zeros(1, dtype=torch.int64, device=DEV)
    pkv.selftest_bounded_wait(20_000, err, waited)          # 20 ms
    assert pkv.get_device_error(err) == pkv.DEVERR_TIMEOUT
    ns = int(waited.item())
    assert 20_000_000 <= ns < 2_000_000_000, ns
    # the device still runs work normally
    x = torch.arange(1024, device=DEV, dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2
