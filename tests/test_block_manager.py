"""The host block manager (pkv_bm_*): prefix reuse, slots, eviction, out of
blocks, and a randomized check of its invariants against a plain model of
what every live sequence holds.  CPU only."""
from __future__ import annotations

import random

import pytest
import torch

import paged_kv_cache_484_b200 as pkv
from paged_kv_cache_484_b200 import build as lib_build

BS = 16


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lib_build.build()


def test_prompt_prefix_reuse_and_slots():
    bm = pkv.BlockManager(16, BS)
    sys_prompt = list(range(100, 140))                  # 40 tokens: 2 full blocks + 8
    assert bm.add_sequence(1, sys_prompt + [1, 2, 3]) == 0
    t1, n1 = bm.block_table(1, 8)
    assert n1 == 43 and (t1[:3] >= 0).all() and (t1[3:] == -1).all()
    # the second request shares the two full blocks, not the partial third
    assert bm.add_sequence(2, sys_prompt + [7, 8]) == 32
    t2, _ = bm.block_table(2, 8)
    assert torch.equal(t2[:2], t1[:2]) and t2[2] != t1[2]
    slots = bm.prompt_slots(2, 42)
    assert (slots[:32] == -1).all()
    assert torch.equal(slots[32:], int(t2[2]) * BS + torch.arange(10))
    # one different token in the first block: nothing shared
    assert bm.add_sequence(3, [999] + sys_prompt[1:]) == 0


def test_append_fills_and_publishes_blocks():
    bm = pkv.BlockManager(8, BS)
    bm.add_sequence(1, list(range(10)))
    t, _ = bm.block_table(1, 4)
    slots = [bm.append(1, 10 + i) for i in range(10)]    # tokens 10..19: block 0 full at 16
    assert slots[:6] == [int(t[0]) * BS + 10 + i for i in range(6)]
    t, n = bm.block_table(1, 4)
    assert n == 20 and slots[6] == int(t[1]) * BS        # token 16 opens the second block
    # the now-full first block serves a new prompt with the same 16 tokens
    assert bm.add_sequence(2, list(range(16)) + [5]) == 16
    assert int(bm.block_table(2, 4)[0][0]) == int(t[0])


def test_free_keeps_blocks_cached_until_needed():
    bm = pkv.BlockManager(4, BS)
    p = list(range(32))
    bm.add_sequence(1, p)                                # 2 full blocks, published
    bm.free_sequence(1)
    assert bm.free_blocks == 4 and bm.cached_blocks == 2
    assert bm.add_sequence(2, p + [1]) == 32              # reused after its owner left
    bm.free_sequence(2)
    # a different prompt that needs every block evicts the cached ones
    bm.add_sequence(3, list(range(500, 564)))
    assert bm.cached_blocks == 4 and bm.free_blocks == 0
    bm.free_sequence(3)
    assert bm.add_sequence(4, p) == 0                     # sequence 1's blocks were evicted


def test_out_of_blocks_is_reported_and_allocates_nothing():
    bm = pkv.BlockManager(3, BS)
    bm.add_sequence(1, list(range(40)))                  # all 3 blocks
    before = bm.free_blocks
    with pytest.raises(pkv.PkvError) as e:
        bm.add_sequence(2, list(range(200, 220)))
    assert e.value.status == 3 and bm.free_blocks == before
    with pytest.raises(pkv.PkvError):
        for i in range(10):                              # fills block 3, then needs a 4th
            bm.append(1, i)
    bm.free_sequence(1)                                  # preempt, then retry
    bm.add_sequence(2, list(range(200, 220)))


def test_bad_arguments():
    bm = pkv.BlockManager(4, BS)
    bm.add_sequence(1, list(range(20)))                  # two blocks
    with pytest.raises(pkv.PkvError):
        bm.add_sequence(1, [4])                          # duplicate id
    with pytest.raises(pkv.PkvError):
        bm.append(7, 1)                                  # unknown sequence
    with pytest.raises(pkv.PkvError):
        bm.free_sequence(7)
    with pytest.raises(pkv.PkvError):
        bm.block_table(1, 1)                             # no room for its second block
    assert bm.shared_tokens(7) == -1


def test_random_operations_keep_the_invariants():
    """Random admissions (prompts drawn from a few shared prefixes), appends
    and frees.  After every step: each live sequence holds ceil(n/16)
    blocks; two live sequences share a block only at the same position and
    only if every token up to the end of that block is the same; blocks in use
    plus available blocks make up the pool."""
    rng = random.Random(7)
    NB = 48
    bm = pkv.BlockManager(NB, BS)
    prefixes = [[rng.randrange(50) for _ in range(rng.choice([16, 33, 48]))] for _ in range(3)]
    live: dict[int, list[int]] = {}
    next_id = 0
    for _ in range(400):
        op = rng.random()
        if op < 0.35 or not live:
            prompt = list(rng.choice(prefixes)) + [rng.randrange(50) for _ in range(rng.randrange(20))]
            try:
                shared = bm.add_sequence(next_id, prompt)
            except pkv.PkvError:
                victim = rng.choice(list(live)) if live else None
                if victim is not None:
                    bm.free_sequence(victim)
                    del live[victim]
                continue
            assert shared % BS == 0 and shared <= len(prompt)
            live[next_id] = prompt
            next_id += 1
        elif op < 0.85:
            sid = rng.choice(list(live))
            tok = rng.randrange(50)
            try:
                bm.append(sid, tok)
                live[sid].append(tok)
            except pkv.PkvError:
                bm.free_sequence(sid)
                del live[sid]
        else:
            sid = rng.choice(list(live))
            bm.free_sequence(sid)
            del live[sid]
        tables = {}
        for sid, toks in live.items():
            row, n = bm.block_table(sid, 64)
            assert n == len(toks)
            nb = (n + BS - 1) // BS
            assert (row[:nb] >= 0).all() and (row[nb:] == -1).all()
            tables[sid] = row[:nb].tolist()
        where = {}
        for sid, blocks in tables.items():
            for j, blk in enumerate(blocks):
                if blk in where:
                    osid, oj = where[blk]
                    assert oj == j, "a block shared at two positions"
                    end = (j + 1) * BS
                    assert live[sid][:end] == live[osid][:end], "a block shared by different prefixes"
                    assert end <= len(live[sid]) and end <= len(live[osid]), "a partial block shared"
                else:
                    where[blk] = (sid, j)
        assert len(where) + bm.free_blocks == NB


def test_prepared_call_marshals_once_and_reports_errors():
    """PreparedCall (the binding's checked-once call) on a host entry point:
    the first call succeeds, the repeat reports the library's status."""
    lib = pkv.load_library()
    bm = pkv.BlockManager(4, BS)
    bm.add_sequence(9, [1, 2, 3])
    call = pkv.PreparedCall(lib, lib.pkv_bm_free_sequence, (bm._h, 9), "pkv_bm_free_sequence", bm)
    call()
    assert bm.free_blocks == 4
    with pytest.raises(pkv.PkvError):
        call()


def test_kv_memory_accounting():
    """Bytes per request and admission capacity, against the element count
    written out by hand: every token holds K and V per kv head per layer, in
    whole 16-token blocks."""
    # Llama-3.2-1B attention: 16 layers, 8 kv heads, head_dim 64, bf16
    per_token = 16 * 2 * 8 * 64 * 2
    assert per_token == 32 * 1024
    assert pkv.kv_request_bytes(16, 8, 64, 2048) == 2048 * per_token == 64 << 20
    assert pkv.kv_request_bytes(16, 8, 64, 2049) == 2064 * per_token   # a 129th block
    assert pkv.kv_request_bytes(16, 8, 64, 0) == 0
    assert pkv.kv_request_bytes(16, 8, 64, 100, kv_dtype=torch.uint8) == 112 * per_token // 2
    assert pkv.kv_request_bytes(32, 8, 128, 1, kv_dtype=torch.float32) == 32 * 2 * 8 * 16 * 128 * 4
    assert pkv.kv_admission_capacity(80 << 30, 16, 8, 64, 2048) == (80 << 30) // (64 << 20)
    assert pkv.kv_admission_capacity((64 << 20) - 1, 16, 8, 64, 2048) == 0
    with pytest.raises(ValueError):
        pkv.kv_request_bytes(0, 8, 64, 10)
    with pytest.raises(ValueError):
        pkv.kv_request_bytes(16, 8, 64, -1)
