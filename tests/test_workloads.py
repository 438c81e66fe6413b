"""The seeded input generator: determinism and the structure each workload promises."""
import torch

from paged_kv_cache_484_b200 import workloads as W


def _check_structure(w: W.Workload):
    B, MB = w.block_tables.shape
    bs = w.block_size
    need = (w.cached_lens.long() + 1 + bs - 1) // bs
    for b in range(B):
        row = w.block_tables[b]
        n = int(need[b])
        assert (row[:n] >= 0).all() and (row[:n] < w.num_blocks).all()
        assert (row[n:] == -1).all()
        L = int(w.cached_lens[b])
        assert int(w.positions[b]) == L
        assert int(w.slot_mapping[b]) == int(row[L // bs]) * bs + L % bs
        assert int(w.decode_lens[b]) == L + 1
    # append slots are distinct and never inside a shared block
    slots = w.slot_mapping.tolist()
    assert len(set(slots)) == len(slots)


def test_config1_and_2_structure_and_determinism():
    for cfg in (1, 2):
        a = W.make_config(cfg)
        b = W.make_config(cfg)
        _check_structure(a)
        for name, t in a.tensors().items():
            assert torch.equal(t, b.tensors()[name]), name
    w1 = W.make_config(1)
    assert w1.num_blocks == 64 and w1.block_tables.shape == (1, 17)
    assert w1.q.dtype == torch.float32 and w1.k_cache.shape == (64, 4, 16, 64)
    w2 = W.make_config(2)
    assert w2.num_blocks == 4096 and w2.block_tables.shape == (1, 129)
    assert w2.k_cache.dtype == torch.bfloat16


def test_private_blocks_are_disjoint_and_prefix_groups_share():
    lens = [10, 40, 2000, 1100, 15, 5000, 31, 1024, 3000]
    w = W.build_workload("t", lens, 4, 2, 16, torch.bfloat16, 1e4, 7, prefix_group=4,
                         prefix_tokens=1024)
    _check_structure(w)
    bs = 16
    owners = {}
    for b, L in enumerate(lens):
        n = (L + 1 + bs - 1) // bs
        shared = min(L // bs, 1024 // bs)
        for j in range(n):
            blk = int(w.block_tables[b, j])
            key = ("shared", b // 4, j) if j < shared else ("private", b, j)
            owners.setdefault(blk, set()).add(key)
    for blk, keys in owners.items():
        assert len(keys) == 1, (blk, keys)   # a physical block has one role
    # sequences of one group agree on their common full prefix blocks
    assert torch.equal(w.block_tables[2, :64], w.block_tables[3, :64])
    assert int(w.block_tables[5, 0]) == int(w.block_tables[7, 0])
    assert int(w.block_tables[0, 0]) != int(w.block_tables[4, 0])   # other group


def test_hot_keys_scaled_by_eight():
    w = W.build_workload("t", [64], 4, 4, 16, torch.bfloat16, 1e4, 3, hot_key_frac=0.25)
    base = W.build_workload("t", [64], 4, 4, 16, torch.bfloat16, 1e4, 3)
    ratio = (w.k_cache.float() / base.k_cache.float())
    ok = (ratio == 1) | (ratio == 8) | (base.k_cache.float() == 0)
    assert ok.all()
    frac = (ratio == 8).float().mean().item()
    assert 0.15 < frac < 0.35
