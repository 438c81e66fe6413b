"""Seeded synthetic inputs for the paged decode step.

This module only draws random numbers and lays out block tables: it holds
none of the attention or RoPE arithmetic, so both the CUDA path and the CPU
oracle can be fed from it.

A workload is one decode step of one layer: every sequence b already holds
``cached_lens[b]`` tokens (positions 0 .. L_b-1, post-RoPE keys) in a paged
cache, and one new token per sequence arrives at position L_b.  The step is
``kv_append`` (rotate q and k of the new token, write k/v into its slot)
followed by ``paged_attention_decode`` over ``L_b + 1`` tokens.

Shapes follow the paged-cache layout used throughout the library:

* ``k_cache``/``v_cache``: [num_blocks, Hkv, block_size, d]
* ``block_tables``: [B, max_blocks] int32, unused entries are -1
* ``q``: [B, Hq, d]; ``k_new``/``v_new``: [B, Hkv, d]
* ``positions``/``slot_mapping``: [B] int64; ``decode_lens``: [B] int32

The five named workloads are the decode shapes of the Llama-3.2-1B-class
serving engines the pages build (32 query / 8 KV heads, head_dim 64, block
size 16), plus a small MHA case and a Llama-3-8B head shape at 128k context.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BLOCK_SIZE = 16


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    block_size: int
    num_blocks: int
    dtype: torch.dtype
    rope_theta: float
    scale: float
    cached_lens: torch.Tensor      # [B] int32, tokens already in the cache
    decode_lens: torch.Tensor      # [B] int32, cached_lens + 1
    block_tables: torch.Tensor     # [B, MB] int32
    positions: torch.Tensor        # [B] int64
    slot_mapping: torch.Tensor     # [B] int64
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    meta: dict = field(default_factory=dict)

    @property
    def max_blocks(self) -> int:
        return self.block_tables.shape[1]

    def tensors(self):
        return dict(q=self.q, k_new=self.k_new, v_new=self.v_new, positions=self.positions,
                    slot_mapping=self.slot_mapping, k_cache=self.k_cache, v_cache=self.v_cache,
                    block_tables=self.block_tables, decode_lens=self.decode_lens)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def build_workload(name: str, cached_lens, Hq: int, Hkv: int, d: int, dtype: torch.dtype,
                   rope_theta: float, seed: int, device="cpu", block_size: int = BLOCK_SIZE,
                   pool_blocks: int | None = None, pool_factor: float = 1.0,
                   prefix_group: int = 0, prefix_tokens: int = 0,
                   hot_key_frac: float = 0.0, hot_key_scale: float = 8.0,
                   table_order=None) -> Workload:
    """Lay out a paged cache for the given cached lengths and fill it with N(0,1).

    * Every sequence needs ceil((L_b + 1) / block_size) blocks: its context plus
      the slot of the token appended this step.
    * With ``prefix_group`` > 1, consecutive groups of that many sequences share
      the physical ids of their first ``prefix_tokens`` tokens, limited to the
      blocks a sequence fills completely (a block that the append writes into
      is always private).
    * Physical ids are a seeded random permutation of the pool, dealt out in
      order, so logical neighbours are scattered.
    * ``hot_key_frac`` of the cached key rows (one row = one token of one KV
      head) are multiplied by ``hot_key_scale`` (exact for powers of two).
    """
    gcpu = _gen("cpu", seed)
    cached = torch.as_tensor(cached_lens, dtype=torch.int64).cpu()
    B = int(cached.numel())
    bs = block_size
    need = (cached + 1 + bs - 1) // bs  # blocks per sequence incl. the append slot
    MB = int(need.max().item()) if B else 1

    # which logical blocks are shared with the group's prefix
    prefix_blocks = prefix_tokens // bs if prefix_group > 1 else 0
    shared = torch.zeros(B, dtype=torch.int64)
    if prefix_blocks:
        shared = torch.minimum(cached // bs, torch.full_like(cached, prefix_blocks))
    n_groups = (B + prefix_group - 1) // prefix_group if prefix_blocks else 0
    private_total = int((need - shared).sum().item())
    shared_total = n_groups * prefix_blocks
    used = private_total + shared_total
    NB = max(int(pool_blocks or 0), int(math.ceil(pool_factor * used)), 1)
    if used > NB:
        raise ValueError(f"pool of {NB} blocks cannot hold {used}")
    perm = torch.randperm(NB, generator=gcpu)
    ids = perm[:used].tolist()

    tables = torch.full((B, MB), -1, dtype=torch.int32)
    cursor = 0
    group_ids = []
    for _ in range(n_groups):
        group_ids.append(ids[cursor:cursor + prefix_blocks])
        cursor += prefix_blocks
    order = range(B) if table_order is None else table_order
    for b in order:
        nb = int(need[b])
        row = []
        ns = int(shared[b])
        if ns:
            row.extend(group_ids[b // prefix_group][:ns])
        row.extend(ids[cursor:cursor + nb - ns])
        cursor += nb - ns
        tables[b, :nb] = torch.tensor(row, dtype=torch.int32)
    assert cursor == used

    positions = cached.clone()
    last_block = tables[torch.arange(B), (cached // bs)].to(torch.int64) if B else cached
    slot_mapping = last_block * bs + cached % bs

    gdev = _gen(device, seed + 7919)
    kw = dict(generator=gdev, device=device, dtype=dtype)
    q = torch.randn((B, Hq, d), **kw)
    k_new = torch.randn((B, Hkv, d), **kw)
    v_new = torch.randn((B, Hkv, d), **kw)
    k_cache = torch.randn((NB, Hkv, bs, d), **kw)
    v_cache = torch.randn((NB, Hkv, bs, d), **kw)
    if hot_key_frac > 0:
        hot = torch.rand((NB, Hkv, bs), generator=gdev, device=device) < hot_key_frac
        k_cache[hot] *= hot_key_scale
        del hot

    return Workload(
        name=name, B=B, Hq=Hq, Hkv=Hkv, d=d, block_size=bs, num_blocks=NB, dtype=dtype,
        rope_theta=float(rope_theta), scale=1.0 / math.sqrt(d),
        cached_lens=cached.to(torch.int32).to(device),
        decode_lens=(cached + 1).to(torch.int32).to(device),
        block_tables=tables.to(device), positions=positions.to(device),
        slot_mapping=slot_mapping.to(device), q=q, k_new=k_new, v_new=v_new,
        k_cache=k_cache, v_cache=v_cache,
        meta=dict(seed=seed, prefix_group=prefix_group, prefix_tokens=prefix_tokens,
                  hot_key_frac=hot_key_frac, pool_factor=pool_factor))


# ---- the five named decode workloads -------------------------------------

CONFIG_NAMES = {
    1: "tiny_mha_fp32_ctx256",
    2: "llama32_1b_layer_decode_b1_ctx2048",
    3: "ragged_batch64_ctx128_4096",
    4: "contbatch256_logctx16_32768_prefix1024x8",
    5: "longctx_b16_ctx131072_d128_splitk",
}


def _uniform_int(g, lo, hi, n):
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int64)


def make_config(cfg: int, device="cpu", num_seqs: int | None = None) -> Workload:
    """Workload ``cfg`` (1..5), seeded with 484 + cfg.  ``num_seqs`` keeps only
    the first that many sequences (the same lengths and layout rules on a
    smaller batch, e.g. for a profiler capture that must stay small); the
    pool and values are then drawn for that batch."""
    seed = 484 + cfg
    name = CONFIG_NAMES[cfg]
    if num_seqs is not None:
        return _truncated(cfg, device, int(num_seqs))
    if cfg == 1:
        # 1 sequence, 4/4 heads, d 64, 256 cached tokens in a 64-block pool, fp32
        return build_workload(name, [256], 4, 4, 64, torch.float32, 1e4, seed, device,
                              pool_blocks=64)
    if cfg == 2:
        # Llama-3.2-1B attention shape, batch 1, 2048 cached tokens, 4096-block pool
        return build_workload(name, [2048], 32, 8, 64, torch.bfloat16, 5e5, seed, device,
                              pool_blocks=4096)
    if cfg == 3:
        g = _gen("cpu", seed + 1)
        lens = _uniform_int(g, 128, 4096, 64)
        return build_workload(name, lens, 32, 8, 64, torch.bfloat16, 5e5, seed, device,
                              pool_factor=1.25)
    if cfg == 4:
        g = _gen("cpu", seed + 1)
        u = torch.rand(256, generator=g, dtype=torch.float64)
        lens = torch.floor(torch.exp(math.log(16) + u * (math.log(32768) - math.log(16))))
        lens = lens.clamp(16, 32768).to(torch.int64)
        return build_workload(name, lens, 32, 8, 64, torch.bfloat16, 5e5, seed, device,
                              pool_factor=1.0, prefix_group=8, prefix_tokens=1024)
    if cfg == 5:
        return build_workload(name, [131072] * 16, 32, 8, 128, torch.bfloat16, 5e5, seed,
                              device, hot_key_frac=0.01, hot_key_scale=8.0)
    raise ValueError(f"unknown config {cfg}")


def _truncated(cfg: int, device, n: int) -> Workload:
    full = {1: ([256], dict(pool_blocks=64)), 2: ([2048], dict(pool_blocks=4096))}
    seed = 484 + cfg
    if cfg in full:
        lens, kw = full[cfg]
        lens = lens[:n]
    elif cfg == 3:
        lens, kw = _uniform_int(_gen("cpu", seed + 1), 128, 4096, 64)[:n], dict(pool_factor=1.25)
    elif cfg == 4:
        g = _gen("cpu", seed + 1)
        u = torch.rand(256, generator=g, dtype=torch.float64)
        lens = torch.floor(torch.exp(math.log(16) + u * (math.log(32768) - math.log(16))))
        lens = lens.clamp(16, 32768).to(torch.int64)[:n]
        kw = dict(pool_factor=1.0, prefix_group=8, prefix_tokens=1024)
    elif cfg == 5:
        lens, kw = [131072] * min(n, 16), dict(hot_key_frac=0.01, hot_key_scale=8.0)
    else:
        raise ValueError(f"unknown config {cfg}")
    shape = {1: (4, 4, 64, torch.float32, 1e4)}.get(
        cfg, (32, 8, 128 if cfg == 5 else 64, torch.bfloat16, 5e5))
    name = f"{CONFIG_NAMES[cfg]}_first{len(lens)}seqs"
    return build_workload(name, lens, *shape, seed, device, **kw)


def config_summary(cfg: int) -> dict:
    """Shape description of a named workload without generating tensors."""
    return {
        1: dict(B=1, Hq=4, Hkv=4, d=64, ctx="256", dtype="f32"),
        2: dict(B=1, Hq=32, Hkv=8, d=64, ctx="2048", dtype="bf16"),
        3: dict(B=64, Hq=32, Hkv=8, d=64, ctx="U[128,4096]", dtype="bf16"),
        4: dict(B=256, Hq=32, Hkv=8, d=64, ctx="logU[16,32768], 8-way shared 1024-token prefix",
                dtype="bf16"),
        5: dict(B=16, Hq=32, Hkv=8, d=128, ctx="131072, 1% keys x8", dtype="bf16"),
    }[cfg]


@dataclass
class SequenceSubset:
    """CPU copy of the inputs that some sequences of a workload need: their
    pages gathered into a compact pool, block tables and slots renumbered to
    it.  Pure data movement; physical ids carry no meaning of their own."""
    seqs: list
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    tables: torch.Tensor
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    positions: torch.Tensor
    slots: torch.Tensor
    decode_lens: torch.Tensor
    theta: float
    scale: float


def e4m3_cache(w: Workload, chunk_blocks: int = 4096):
    """The workload's cached K/V as an 8-bit cache: one scale per tensor
    (max |x| / 448, so the largest value maps to the largest E4M3 number) and
    PyTorch's float8_e4m3fn cast of x / scale, as uint8 codes; the V pages
    transposed to [num_blocks, Hkv, d, block_size].  Returns (k_cache,
    v_cache, k_scale, v_scale); the cast is PyTorch's, not the library's."""
    def amax(t):
        return max(float(t[i:i + chunk_blocks].float().abs().max())
                   for i in range(0, t.shape[0], chunk_blocks))

    ks, vs = amax(w.k_cache) / 448.0, amax(w.v_cache) / 448.0
    NB, Hkv, bs, d = w.k_cache.shape
    k8 = torch.empty((NB, Hkv, bs, d), dtype=torch.uint8, device=w.k_cache.device)
    v8 = torch.empty((NB, Hkv, d, bs), dtype=torch.uint8, device=w.v_cache.device)
    for i in range(0, NB, chunk_blocks):
        j = min(NB, i + chunk_blocks)
        k8[i:j] = (w.k_cache[i:j].float() / ks).to(torch.float8_e4m3fn).view(torch.uint8)
        v8[i:j] = (w.v_cache[i:j].float() / vs).to(torch.float8_e4m3fn).view(torch.uint8) \
            .transpose(2, 3)
    return k8, v8, ks, vs


def e4m3_pack(k8: torch.Tensor, v8: torch.Tensor) -> torch.Tensor:
    """The 8-bit cache as the library stores it: K codes [NB, Hkv, 16, d] and
    transposed V codes [NB, Hkv, d, 16] interleaved page by page into one
    uint8 buffer [NB, Hkv, 2, 16 * d] (each page's K half, then its V half).
    Pure data movement."""
    NB, Hkv = k8.shape[:2]
    return torch.stack((k8.reshape(NB, Hkv, -1), v8.reshape(NB, Hkv, -1)), dim=2).contiguous()


def e4m3_halves(kv8: torch.Tensor):
    """Views of a packed 8-bit cache: (K [NB, Hkv, 16, d], V [NB, Hkv, d, 16]);
    they alias kv8 and are not contiguous (use .contiguous() for a copy)."""
    NB, Hkv, _, pg = kv8.shape
    d = pg // BLOCK_SIZE
    return kv8[:, :, 0].view(NB, Hkv, BLOCK_SIZE, d), kv8[:, :, 1].view(NB, Hkv, d, BLOCK_SIZE)


def extract_sequences(w: Workload, seqs) -> SequenceSubset:
    """Copy the inputs of sequences ``seqs`` to the host (read before any step
    modifies the workload's tensors)."""
    seqs = list(seqs)
    bs = w.block_size
    rows = []
    for b in seqs:
        n = (int(w.cached_lens[b]) + 1 + bs - 1) // bs
        rows.append(w.block_tables[b, :n].to(torch.int64))
    ids = torch.cat(rows)
    uniq, inv = torch.unique(ids, return_inverse=True)
    MB = max(r.numel() for r in rows)
    tables = torch.full((len(seqs), MB), -1, dtype=torch.int32)
    off = 0
    for i, r in enumerate(rows):
        tables[i, :r.numel()] = inv[off:off + r.numel()].to(torch.int32).cpu()
        off += r.numel()
    sel = torch.tensor(seqs, device=w.q.device)
    cached = w.cached_lens[sel].cpu().to(torch.int64)
    slots = tables[torch.arange(len(seqs)), (cached // bs)].to(torch.int64) * bs + cached % bs
    return SequenceSubset(
        seqs=seqs, k_cache=w.k_cache[uniq].cpu(), v_cache=w.v_cache[uniq].cpu(), tables=tables,
        q=w.q[sel].cpu(), k_new=w.k_new[sel].cpu(), v_new=w.v_new[sel].cpu(),
        positions=w.positions[sel].cpu(), slots=slots, decode_lens=w.decode_lens[sel].cpu(),
        theta=w.rope_theta, scale=w.scale)
