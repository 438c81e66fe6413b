"""Pins for the fp64 CPU oracle.

The oracle is what the CUDA path is checked against, so it is itself checked
against things it does not compute: library routines that reduce to the same
definition (PyTorch's fp64 scaled-dot-product attention, Hugging Face's Llama
RoPE, PyTorch's float32->bf16 cast), closed forms of the softmax, the
invariants the pages state (paged == contiguous, decode == last row of the
full-prefix causal pass, chunked == full prefix), and exact arithmetic on tiny
inputs.  Every pin is a plain function of an ``Oracle`` so that
``test_planted_mistake_is_caught`` can run the whole set against deliberately
broken copies of the oracle and show that each plausible mistake fails one.
"""
from __future__ import annotations

import decimal
import math

import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import Oracle, OracleError, build as oracle_build

# ---------------------------------------------------------------- helpers


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def sdpa(q, K, V, scale, causal=False):
    """PyTorch fp64 SDPA.  q [Lq, Hq, d], K/V [L, Hkv, d]; kv head j serves
    query heads j*G .. j*G+G-1 (repeat_interleave, the Llama repeat_kv order)."""
    Hq, Hkv = q.shape[1], K.shape[1]
    G = Hq // Hkv
    Kr = K.repeat_interleave(G, dim=1)
    Vr = V.repeat_interleave(G, dim=1)
    out = F.scaled_dot_product_attention(
        q.permute(1, 0, 2)[None], Kr.permute(1, 0, 2)[None], Vr.permute(1, 0, 2)[None],
        scale=scale, is_causal=causal)
    return out[0].permute(1, 0, 2)


def random_paged(lens, Hkv, d, bs, dtype, seed, extra_blocks=3):
    """Contiguous per-sequence K/V plus the same data scattered into a paged
    pool through a random block table (layout [NB, Hkv, bs, d])."""
    g = _gen(seed)
    need = [max(1, (L + bs - 1) // bs) for L in lens]
    NB = sum(need) + extra_blocks
    perm = torch.randperm(NB, generator=g)
    MB = max(need)
    tables = torch.full((len(lens), MB), -1, dtype=torch.int32)
    kpool = torch.randn(NB, Hkv, bs, d, generator=g).to(dtype)
    vpool = torch.randn(NB, Hkv, bs, d, generator=g).to(dtype)
    Ks, Vs, c = [], [], 0
    for b, L in enumerate(lens):
        ids = perm[c:c + need[b]]
        c += need[b]
        tables[b, :need[b]] = ids.to(torch.int32)
        K = torch.randn(L, Hkv, d, generator=g).to(dtype)
        V = torch.randn(L, Hkv, d, generator=g).to(dtype)
        for t in range(L):
            kpool[ids[t // bs], :, t % bs, :] = K[t]
            vpool[ids[t // bs], :, t % bs, :] = V[t]
        Ks.append(K)
        Vs.append(V)
    return kpool, vpool, tables, Ks, Vs


def assert_close(a, b, tol, what=""):
    err = (a - b).abs().max().item() if a.numel() else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- pins
# Each pin takes an Oracle and raises AssertionError on a mismatch.


def pin_round_bf16_matches_torch_cast(orc: Oracle):
    """float32 values rounded to bf16 in one step must equal PyTorch's
    float32 -> bfloat16 cast (round to nearest even), across the exponent
    range, subnormals included."""
    g = _gen(1)
    mant = torch.randn(20000, generator=g, dtype=torch.float64)
    expo = torch.randint(-140, 120, (20000,), generator=g).to(torch.float64)
    x32 = (mant * torch.pow(2.0, expo)).to(torch.float32)
    x32 = x32[torch.isfinite(x32)]
    want = x32.to(torch.bfloat16).view(torch.int16)
    got = orc.round_bf16(x32.to(torch.float64)).view(torch.int16)
    bad = (want != got).nonzero()
    assert bad.numel() == 0, f"{bad.numel()} mismatches, first at {x32[bad[0]].item()!r}"


def pin_round_bf16_single_rounding(orc: Oracle):
    """Ties go to even, and a double just above a bf16 midpoint rounds up even
    though going through float32 first would land exactly on the midpoint."""
    cases = [
        (1.0 + 2.0**-8, 0x3F80),                  # tie -> even (1.0)
        (1.0 + 3 * 2.0**-8, 0x3F82),              # tie -> even (1 + 2^-6)
        (1.0 + 2.0**-8 + 2.0**-40, 0x3F81),       # above the tie: up
        (-(1.0 + 2.0**-8), 0xBF80),
        (2.0**-134, 0x0000),                      # half the subnormal spacing -> 0
        (3 * 2.0**-134, 0x0002),                  # 1.5 spacings -> 2 (even)
        ((2 - 2.0**-7) * 2.0**127, 0x7F7F),       # largest finite
        ((2 - 2.0**-8) * 2.0**127, 0x7F80),       # rounds past it -> inf
        (0.0, 0x0000),
    ]
    x = torch.tensor([c[0] for c in cases], dtype=torch.float64)
    got = orc.round_bf16(x).view(torch.int16).to(torch.int64) & 0xFFFF
    for (v, want), bits in zip(cases, got.tolist()):
        assert bits == want, f"round_bf16({v!r}) = {bits:#06x}, want {want:#06x}"


def pin_bf16_widening_exact(orc: Oracle):
    bits = torch.arange(0, 65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    want = bits.to(torch.float64)
    got = orc.bf16_to_double(bits)
    fin = torch.isfinite(want)
    assert torch.equal(got[fin], want[fin])
    assert torch.equal(torch.isnan(got), torch.isnan(want))


def pin_rope_position_zero_is_identity(orc: Oracle):
    x = torch.randn(5, 64, generator=_gen(2), dtype=torch.float64)
    y = orc.rope(x, torch.zeros(5, dtype=torch.int64), 1e4)
    assert torch.equal(x, y)


def pin_rope_matches_hf_llama(orc: Oracle):
    """Rotate-half pairing, sign and theta^(-2i/d) frequencies, against
    Hugging Face's Llama rotary embedding (float32, so small positions)."""
    from transformers import LlamaConfig
    from transformers.models.llama import modeling_llama as hf

    for d, theta in ((64, 1e4), (128, 5e5), (64, 5e5)):
        cfg = LlamaConfig(hidden_size=4 * d, num_attention_heads=4, num_key_value_heads=4,
                          head_dim=d, rope_theta=theta)
        rot = hf.LlamaRotaryEmbedding(cfg)
        pos = torch.arange(0, 48, dtype=torch.int64)
        x = torch.randn(len(pos), d, generator=_gen(3), dtype=torch.float64)
        cos, sin = rot(x.to(torch.float32)[None], pos[None])
        xq = x.to(torch.float32)[None, None]      # [1, 1, n, d]
        ref, _ = hf.apply_rotary_pos_emb(xq, xq, cos, sin)
        got = orc.rope(x, pos, theta)
        assert_close(got, ref[0, 0].to(torch.float64), 2e-5, f"rope vs HF d={d}")


def pin_rope_is_complex_rotation(orc: Oracle):
    """(x_i, x_{i+d/2}) as the complex number x_i + j x_{i+d/2} is multiplied by
    exp(j * pos * theta^(-2i/d)) -- a rotation, so norms and relative
    positions are preserved, and rotations compose."""
    d, theta = 64, 5e5
    g = _gen(4)
    x = torch.randn(6, d, generator=g, dtype=torch.float64)
    pos = torch.tensor([0, 1, 17, 255, 4096, 131072], dtype=torch.int64)
    got = orc.rope(x, pos, theta)
    i = torch.arange(d // 2, dtype=torch.float64)
    freq = theta ** (-2.0 * i / d)
    z = torch.complex(x[:, : d // 2], x[:, d // 2:])
    zr = z * torch.exp(1j * pos[:, None].to(torch.float64) * freq[None])
    want = torch.cat([zr.real, zr.imag], dim=1)
    assert_close(got, want, 1e-11, "rope vs complex rotation")
    # pair norms preserved
    n0 = x[:, : d // 2] ** 2 + x[:, d // 2:] ** 2
    n1 = got[:, : d // 2] ** 2 + got[:, d // 2:] ** 2
    assert_close(n0, n1, 1e-11, "pair norms")
    # composition: rope(rope(x, m), n) == rope(x, m + n)
    m = torch.tensor([3, 100, 5000, 7, 0, 9], dtype=torch.int64)
    n = torch.tensor([4, 28, 1, 2000, 11, 0], dtype=torch.int64)
    assert_close(orc.rope(orc.rope(x, m, theta), n, theta), orc.rope(x, m + n, theta), 1e-9,
                 "composition")
    # relative position: <rope(q, a), rope(k, b)> depends on a - b only
    q = torch.randn(1, d, generator=g, dtype=torch.float64)
    k = torch.randn(1, d, generator=g, dtype=torch.float64)

    def dot(a, b):
        return (orc.rope(q, torch.tensor([a]), theta) * orc.rope(k, torch.tensor([b]), theta)).sum()

    base = dot(5, 2)
    for shift in (1, 100, 9999):
        assert abs(dot(5 + shift, 2 + shift) - base) < 1e-9 * (1 + abs(base))


def pin_decode_matches_sdpa(orc: Oracle):
    """Paged decode equals PyTorch's fp64 SDPA over the gathered context, for
    MHA and GQA groups, ragged lengths and both storage types."""
    for (Hq, Hkv, d, dtype, lens, seed) in [
        (4, 4, 64, torch.float32, [1, 15, 16, 17, 40], 10),
        (8, 2, 16, torch.bfloat16, [33, 1, 64], 11),
        (8, 1, 8, torch.bfloat16, [5, 48], 12),
        (16, 2, 64, torch.float32, [31], 13),
    ]:
        bs = 16
        kpool, vpool, tables, Ks, Vs = random_paged(lens, Hkv, d, bs, dtype, seed)
        q = torch.randn(len(lens), Hq, d, generator=_gen(seed + 100)).to(dtype)
        scale = 1.0 / math.sqrt(d)
        ctx = torch.tensor(lens, dtype=torch.int32)
        got = orc.paged_attention_decode(q, kpool, vpool, tables, ctx, scale)
        for b, L in enumerate(lens):
            want = sdpa(q[b:b + 1].double(), Ks[b].double(), Vs[b].double(), scale)[0]
            assert_close(got[b], want, 1e-12, f"decode vs SDPA b={b} L={L}")


def pin_decode_is_last_row_of_causal_prefill(orc: Oracle):
    """Decode of the last token over the cached prefix equals the last row of
    the full-prefix causal pass; the causal pass itself equals SDPA(causal)."""
    g = _gen(20)
    L, Hq, Hkv, d = 37, 8, 2, 16
    Q = torch.randn(L, Hq, d, generator=g, dtype=torch.float64)
    K = torch.randn(L, Hkv, d, generator=g, dtype=torch.float64)
    V = torch.randn(L, Hkv, d, generator=g, dtype=torch.float64)
    scale = 0.3
    full = orc.causal_prefill(Q, K, V, scale)
    assert_close(full, sdpa(Q, K, V, scale, causal=True), 1e-12, "causal vs SDPA")
    for r in (0, 1, 16, L - 1):
        dec = orc.contiguous_decode(Q[r], K[: r + 1], V[: r + 1], scale)
        assert_close(dec, full[r], 1e-12, f"decode vs causal row {r}")


def pin_paged_equals_contiguous(orc: Oracle):
    lens = [70, 3, 16]
    Hq, Hkv, d = 8, 4, 32
    kpool, vpool, tables, Ks, Vs = random_paged(lens, Hkv, d, 16, torch.float32, 21)
    q = torch.randn(len(lens), Hq, d, generator=_gen(22))
    got = orc.paged_attention_decode(q, kpool, vpool, tables, torch.tensor(lens, dtype=torch.int32), 0.2)
    for b in range(len(lens)):
        want = orc.contiguous_decode(q[b].double(), Ks[b].double(), Vs[b].double(), 0.2)
        assert_close(got[b], want, 1e-12, f"paged vs contiguous b={b}")


def pin_block_relabel_invariance(orc: Oracle):
    """Relabelling physical block ids (pool and table together) changes nothing."""
    lens = [50, 9]
    kpool, vpool, tables, _, _ = random_paged(lens, 2, 16, 16, torch.bfloat16, 23, extra_blocks=5)
    q = torch.randn(2, 4, 16, generator=_gen(24)).to(torch.bfloat16)
    ctx = torch.tensor(lens, dtype=torch.int32)
    a = orc.paged_attention_decode(q, kpool, vpool, tables, ctx, 0.25)
    NB = kpool.shape[0]
    pi = torch.randperm(NB, generator=_gen(25))
    k2 = torch.empty_like(kpool)
    v2 = torch.empty_like(vpool)
    k2[pi] = kpool
    v2[pi] = vpool
    t2 = torch.where(tables >= 0, pi[tables.clamp(min=0).long()].to(torch.int32), tables)
    b = orc.paged_attention_decode(q, k2, v2, t2, ctx, 0.25)
    assert torch.equal(a, b)


def _single(orc, q, K, V, scale, dtype=torch.float64):
    """Run the paged decode for one sequence laid out in one block per 16 tokens."""
    L, Hkv, d = K.shape
    nb = max(1, (L + 15) // 16)
    kpool = torch.zeros(nb, Hkv, 16, d, dtype=torch.float32)
    vpool = torch.zeros(nb, Hkv, 16, d, dtype=torch.float32)
    for t in range(L):
        kpool[t // 16, :, t % 16] = K[t].to(torch.float32)
        vpool[t // 16, :, t % 16] = V[t].to(torch.float32)
    tables = torch.arange(nb, dtype=torch.int32)[None]
    return orc.paged_attention_decode(q[None].to(torch.float32), kpool, vpool, tables,
                                      torch.tensor([L], dtype=torch.int32), scale)[0]


def pin_closed_forms(orc: Oracle):
    g = _gen(30)
    d, Hq, Hkv = 8, 4, 2
    q = torch.randn(Hq, d, generator=g)
    # one token: the output is that token's V, exactly
    K = torch.randn(1, Hkv, d, generator=g)
    V = torch.randn(1, Hkv, d, generator=g)
    out = _single(orc, q, K, V, 0.7)
    assert torch.equal(out, V[0].repeat_interleave(2, 0).double())
    # identical keys: uniform weights, output = mean of V
    L = 23
    K = torch.randn(1, Hkv, d, generator=g).expand(L, Hkv, d).contiguous()
    V = torch.randn(L, Hkv, d, generator=g)
    out = _single(orc, q, K, V, 0.7)
    assert_close(out, V.double().mean(0).repeat_interleave(2, 0), 1e-12, "identical keys")
    # zero scale: uniform weights as well
    K = torch.randn(L, Hkv, d, generator=g)
    out = _single(orc, q, K, V, 0.0)
    assert_close(out, V.double().mean(0).repeat_interleave(2, 0), 1e-12, "scale 0")
    # all-ones V: the weights sum to one
    out = _single(orc, q, K, torch.ones(L, Hkv, d), 0.9)
    assert_close(out, torch.ones_like(out), 1e-15 * L, "weights sum to 1")
    # one key far more aligned with q than the rest: output = that token's V
    K = torch.randn(L, Hkv, d, generator=g) * 0.01
    K[11] = torch.cat([q[0:1], q[2:3]], 0) * 1e3
    out = _single(orc, q, K, V, 1.0)
    assert_close(out[0], V[11, 0].double(), 1e-9, "dominant key")
    assert_close(out[2], V[11, 1].double(), 1e-9, "dominant key")
    # two tokens whose scores differ by ln 3: weights 1/4 and 3/4
    kp = torch.zeros(1, 1, 16, 4)
    vp = torch.zeros(1, 1, 16, 4)
    kp[0, 0, 1, 0] = 1.0            # s_0 = 0, s_1 = scale = ln 3
    vp[0, 0, 0, 0] = 4.0
    vp[0, 0, 1, 1] = 4.0
    qq = torch.tensor([[[1.0, 0.0, 0.0, 0.0]]])
    out = orc.paged_attention_decode(qq, kp, vp, torch.zeros(1, 1, dtype=torch.int32),
                                     torch.tensor([2], dtype=torch.int32), math.log(3.0))
    assert_close(out[0, 0], torch.tensor([1.0, 3.0, 0, 0], dtype=torch.float64), 1e-14, "ln3")


def pin_gqa_group_mapping(orc: Oracle):
    """Query head h reads kv head h // G: with V = kvhead index, every query
    head's output is its group's index."""
    Hq, Hkv, d, L = 8, 4, 16, 20
    g = _gen(31)
    K = torch.randn(L, Hkv, d, generator=g)
    V = torch.arange(Hkv, dtype=torch.float32)[None, :, None].expand(L, Hkv, d).contiguous()
    q = torch.randn(Hq, d, generator=g)
    out = _single(orc, q, K, V, 0.5)
    want = (torch.arange(Hq) // (Hq // Hkv)).double()[:, None].expand(Hq, d)
    assert_close(out, want, 1e-13, "group mapping")


def pin_empty_context(orc: Oracle):
    q = torch.randn(2, 4, 8, generator=_gen(32))
    kp = torch.full((2, 2, 16, 8), float("nan"))
    out = orc.paged_attention_decode(q, kp, kp.clone(), torch.zeros(2, 1, dtype=torch.int32),
                                     torch.tensor([0, 0], dtype=torch.int32), 0.5)
    assert torch.equal(out, torch.zeros_like(out))


def pin_exact_arithmetic_tiny(orc: Oracle):
    """Small integer inputs against a 60-digit decimal evaluation."""
    decimal.getcontext().prec = 60
    D = decimal.Decimal
    g = _gen(33)
    for L in (1, 2, 5, 8):
        q = torch.randint(-3, 4, (1, 4), generator=g).float()
        K = torch.randint(-3, 4, (L, 1, 4), generator=g).float()
        V = torch.randint(-5, 6, (L, 1, 4), generator=g).float()
        scale = 0.5
        out = _single(orc, q, K, V, scale)
        s = [D(scale) * sum(D(int(q[0, i])) * D(int(K[t, 0, i])) for i in range(4)) for t in range(L)]
        w = [x.exp() for x in s]
        tot = sum(w)
        for i in range(4):
            want = sum(w[t] * D(int(V[t, 0, i])) for t in range(L)) / tot
            got = out[0, i].item()
            assert math.isfinite(got), (L, i, got)
            assert abs(D(got) - want) < D("1e-14"), (L, i)


def _append_case(dtype, seed):
    g = _gen(seed)
    T, Hq, Hkv, d, NB, bs = 5, 8, 2, 16, 6, 16
    q = torch.randn(T, Hq, d, generator=g).to(dtype)
    k = torch.randn(T, Hkv, d, generator=g).to(dtype)
    v = torch.randn(T, Hkv, d, generator=g).to(dtype)
    pos = torch.tensor([0, 7, 300, 4095, 131072], dtype=torch.int64)
    slots = torch.tensor([3, -1, 16 * 4 + 15, 17, 16 * 5], dtype=torch.int64)
    return q, k, v, pos, slots, NB, bs


def pin_append_placement_and_values(orc: Oracle):
    """After the append exactly the addressed rows change; v is copied bit for
    bit; k and q are the complex rotation of the inputs rounded once."""
    for dtype, sentinel_bits in ((torch.bfloat16, 0x7B7B), (torch.float32, 0x7B7B7B7B)):
        q, k, v, pos, slots, NB, bs = _append_case(dtype, 40)
        T, Hq, d = q.shape
        Hkv = k.shape[1]
        itype = torch.int16 if dtype == torch.bfloat16 else torch.int32
        sent = torch.full((NB, Hkv, bs, d), sentinel_bits, dtype=itype).view(dtype)
        kc, vc = sent.clone(), sent.clone()
        q2 = q.clone()
        orc.kv_append(q2, k.clone(), v.clone(), pos, slots, kc, vc, 5e5)
        changed = (kc.view(itype) != sent.view(itype)) | (vc.view(itype) != sent.view(itype))
        want_rows = torch.zeros(NB, Hkv, bs, dtype=torch.bool)
        for t, s in enumerate(slots.tolist()):
            if s >= 0:
                want_rows[s // bs, :, s % bs] = True
        assert torch.equal(changed.any(-1), want_rows), "rows written"
        assert not (changed.any(-1) ^ changed.all(-1)).any(), "partial rows"

        def rot(x, p):  # complex-form rotation, fp64, per token
            i = torch.arange(d // 2, dtype=torch.float64)
            z = torch.complex(x[..., : d // 2].double(), x[..., d // 2:].double())
            z = z * torch.exp(1j * float(p) * 5e5 ** (-2.0 * i / d))
            return torch.cat([z.real, z.imag], -1)

        for t, s in enumerate(slots.tolist()):
            if dtype == torch.bfloat16:
                want_q = orc.round_bf16(rot(q[t], pos[t]))
            else:
                want_q = rot(q[t], pos[t]).to(torch.float32)
            diff = (q2[t].double() - want_q.double()).abs().max().item()
            assert diff <= (1e-6 if dtype == torch.float32 else 0.0), f"q token {t}: {diff}"
            if s < 0:
                continue
            assert torch.equal(vc[s // bs, :, s % bs].view(itype), v[t].view(itype)), "v bits"
            if dtype == torch.bfloat16:
                want_k = orc.round_bf16(rot(k[t], pos[t]))
                assert torch.equal(kc[s // bs, :, s % bs].view(itype), want_k.view(itype)), "k"
            else:
                assert_close(kc[s // bs, :, s % bs].double(), rot(k[t], pos[t]), 1e-6, "k f32")


def pin_append_rejects_out_of_range_slot(orc: Oracle):
    q, k, v, pos, slots, NB, bs = _append_case(torch.float32, 41)
    slots[2] = NB * bs
    kc = torch.zeros(NB, k.shape[1], bs, k.shape[2])
    vc = torch.zeros_like(kc)
    q0 = q.clone()
    try:
        orc.kv_append(q, k, v, pos, slots, kc, vc, 1e4)
    except OracleError:
        pass
    else:
        raise AssertionError("out-of-range slot accepted")
    assert torch.equal(q, q0) and not kc.any() and not vc.any(), "partial write before the error"


def pin_append_then_decode_is_causal_last_row(orc: Oracle):
    """Chunked equals full prefix: L cached tokens plus one appended token,
    decoded over L + 1 tokens, equal the last row of a causal pass over the
    whole sequence (the appended key rotated, the cached ones taken as is)."""
    g = _gen(42)
    L, Hq, Hkv, d, bs = 45, 8, 2, 16, 16
    theta = 1e4
    K = torch.randn(L, Hkv, d, generator=g)
    V = torch.randn(L, Hkv, d, generator=g)
    nb = (L + 1 + bs - 1) // bs
    ids = torch.randperm(nb + 2, generator=g)[:nb]
    kc = torch.zeros(nb + 2, Hkv, bs, d)
    vc = torch.zeros_like(kc)
    for t in range(L):
        kc[ids[t // bs], :, t % bs] = K[t]
        vc[ids[t // bs], :, t % bs] = V[t]
    q = torch.randn(1, Hq, d, generator=g)
    kn = torch.randn(1, Hkv, d, generator=g)
    vn = torch.randn(1, Hkv, d, generator=g)
    slot = torch.tensor([int(ids[L // bs]) * bs + L % bs])
    pos = torch.tensor([L])
    q_rot = q.clone()
    orc.kv_append(q_rot, kn.clone(), vn.clone(), pos, slot, kc, vc, theta)
    out = orc.paged_attention_decode(q_rot, kc, vc, ids[None].to(torch.int32),
                                     torch.tensor([L + 1], dtype=torch.int32), 1 / math.sqrt(d))
    i = torch.arange(d // 2, dtype=torch.float64)
    ang = L * theta ** (-2.0 * i / d)

    def rot(x):
        z = torch.complex(x[..., : d // 2].double(), x[..., d // 2:].double()) * torch.exp(1j * ang)
        return torch.cat([z.real, z.imag], -1).to(torch.float32).double()

    K_all = torch.cat([K.double(), rot(kn)], 0)
    V_all = torch.cat([V.double(), vn.double()], 0)
    Q_all = torch.randn(L + 1, Hq, d, generator=g, dtype=torch.float64)
    Q_all[L] = rot(q[0])
    want = sdpa(Q_all, K_all, V_all, 1 / math.sqrt(d), causal=True)[L]
    assert_close(out[0], want, 1e-6, "append+decode vs causal")  # q/k rounded to f32


def pin_chunked_prefill_matches_causal_sdpa(orc: Oracle):
    """A prefill chunk (the last C tokens of each sequence) over the paged
    cache equals PyTorch's fp64 causal SDPA over the gathered context, rows
    L-C .. L-1; and a chunk of the whole context equals the oracle's own
    full-prefix causal pass."""
    for (Hq, Hkv, d, lens, C, seed) in [(8, 2, 16, [40, 17, 5], 5, 30),
                                        (4, 4, 8, [33], 33, 31),
                                        (8, 1, 16, [64, 20], 1, 32)]:
        kpool, vpool, tables, Ks, Vs = random_paged(lens, Hkv, d, 16, torch.float32, seed)
        B = len(lens)
        q = torch.randn(B, C, Hq, d, generator=_gen(seed + 100))
        scale = 1.0 / math.sqrt(d)
        got = orc.paged_chunked_prefill(q, kpool, vpool, tables,
                                        torch.tensor(lens, dtype=torch.int32), scale)
        for b, L in enumerate(lens):
            Q_all = torch.zeros(L, Hq, d, dtype=torch.float64)
            Q_all[L - C:] = q[b].double()
            want = sdpa(Q_all, Ks[b].double(), Vs[b].double(), scale, causal=True)[L - C:]
            assert_close(got[b], want, 1e-12, f"chunked prefill vs causal SDPA b={b}")
            if C == L:
                full = orc.causal_prefill(q[b].double(), Ks[b].double(), Vs[b].double(), scale)
                assert_close(got[b], full, 1e-12, "whole-context chunk vs causal pass")



# ---------------------------------------------------------------- 8-bit cache


def _e4m3_value(codes):
    """PyTorch's own reading of E4M3 codes (float8_e4m3fn), as float64."""
    return codes.view(torch.float8_e4m3fn).to(torch.float64)


def pin_e4m3_decode_matches_torch(orc: Oracle):
    """Every one of the 256 codes means what PyTorch's float8_e4m3fn says
    (the OCP E4M3 format: bias 7, subnormals m * 2^-9, S.1111.111 NaN)."""
    c = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    got, want = orc.e4m3_to_double(c), _e4m3_value(c)
    same = (got == want) | (got.isnan() & want.isnan())
    assert bool(same.all()), f"codes {c[~same].tolist()} decode differently"
    assert got[0x7E].item() == 448.0 and got[0x01].item() == 2.0 ** -9


def pin_e4m3_round_matches_torch_cast(orc: Oracle):
    """Rounding binary32 values to E4M3 equals PyTorch's float32 -> float8
    cast (nearest, ties to even) across the range, subnormals and exact
    midpoints between neighbouring codes included; beyond the range the
    oracle saturates to +-448."""
    g = _gen(61)
    mant = torch.randn(50000, generator=g, dtype=torch.float64)
    expo = torch.randint(-14, 10, (50000,), generator=g).to(torch.float64)
    x = (mant * torch.pow(2.0, expo)).to(torch.float32).to(torch.float64)
    vals = _e4m3_value(torch.arange(0, 0x7E, dtype=torch.int32).to(torch.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    x = torch.cat([x, mids, -mids, vals, -vals]).clamp(-464.0, 464.0)
    got = orc.round_e4m3(x)
    want = x.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
    bad = (got != want).nonzero()
    assert bad.numel() == 0, f"{bad.numel()} mismatches, first at {x[bad[0]].item()!r}"
    big = torch.tensor([470.0, 1e6, float("inf"), -500.0, -float("inf")], dtype=torch.float64)
    assert orc.round_e4m3(big).tolist() == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE], "saturation"


def pin_e4m3_quantizer_rounds_through_binary32(orc: Oracle):
    """The cache quantizer decides in binary32: v / v_scale that lies just
    above the midpoint between 1 and 1.125 in double, but rounds onto it in
    binary32, goes to 1 (even); rounded from the double directly it would
    go to 1.125."""
    x = torch.tensor([1.0625 + 2.0 ** -40], dtype=torch.float64)
    assert orc.round_e4m3(x).tolist() == [0x39], "double rounding of the rounding itself"
    T, Hq, Hkv, d, NB, bs = 1, 1, 1, 2, 1, 16
    q = torch.zeros(T, Hq, d)
    k = torch.zeros(T, Hkv, d)
    v = torch.full((T, Hkv, d), 1.0625)
    kc = torch.zeros(NB, Hkv, bs, d, dtype=torch.uint8)
    vc = torch.zeros(NB, Hkv, d, bs, dtype=torch.uint8)
    v_scale = 1.0 - 2.0 ** -40  # v / v_scale = 1.0625 + ~1e-12
    orc.kv_append_e4m3(q, k, v, torch.tensor([0]), torch.tensor([3]), kc, vc, 1e4, 1.0, v_scale)
    assert vc[0, 0, :, 3].tolist() == [0x38, 0x38], vc[0, 0, :, 3].tolist()


def _random_e4m3_cache(lens, Hkv, d, bs, seed, extra_blocks=3):
    """Random finite codes in a paged pool (k [NB, Hkv, bs, d], v transposed
    [NB, Hkv, d, bs]) and the per-sequence code rows [L, Hkv, d]."""
    g = _gen(seed)
    need = [max(1, (L + bs - 1) // bs) for L in lens]
    NB = sum(need) + extra_blocks
    perm = torch.randperm(NB, generator=g)
    tables = torch.full((len(lens), max(need)), -1, dtype=torch.int32)

    def codes(*shape):
        c = torch.randint(0, 256, shape, generator=g, dtype=torch.int32).to(torch.uint8)
        return torch.where((c & 0x7F) == 0x7F, c ^ 0x01, c)  # no NaN codes

    kc, vc = codes(NB, Hkv, bs, d), codes(NB, Hkv, d, bs)
    Ks, Vs, c0 = [], [], 0
    for b, L in enumerate(lens):
        ids = perm[c0:c0 + need[b]]
        c0 += need[b]
        tables[b, :need[b]] = ids.to(torch.int32)
        K, V = codes(L, Hkv, d), codes(L, Hkv, d)
        for t in range(L):
            kc[ids[t // bs], :, t % bs, :] = K[t]
            vc[ids[t // bs], :, :, t % bs] = V[t]
        Ks.append(K)
        Vs.append(V)
    return kc, vc, tables, Ks, Vs


def pin_e4m3_decode_matches_sdpa_over_dequantized(orc: Oracle):
    """Decode over the 8-bit cache equals PyTorch's fp64 SDPA over the
    dequantized contiguous K/V (code value x scale); with power-of-two
    scales it also equals the oracle's own fp32-cache decode over the same
    values, which are exact in fp32."""
    for (Hq, Hkv, d, lens, ks, vs, seed) in [(8, 2, 16, [40, 17, 1, 33], 0.0123, 0.0311, 70),
                                             (4, 4, 8, [5, 16], 0.125, 0.0625, 71)]:
        kc, vc, tables, Ks, Vs = _random_e4m3_cache(lens, Hkv, d, 16, seed)
        B = len(lens)
        q = torch.randn(B, Hq, d, generator=_gen(seed + 1)).to(torch.bfloat16)
        scale = 1.0 / math.sqrt(d)
        cl = torch.tensor(lens, dtype=torch.int32)
        got = orc.paged_attention_decode_e4m3(q, kc, vc, tables, cl, scale, ks, vs)
        for b in range(B):
            K = _e4m3_value(Ks[b]) * ks
            V = _e4m3_value(Vs[b]) * vs
            want = sdpa(q[b][None].double(), K, V, scale)[0]
            assert_close(got[b], want, 1e-12, f"e4m3 decode vs SDPA b={b}")
        if ks == 0.125:
            kf = (_e4m3_value(kc) * ks).to(torch.float32)
            vf = (_e4m3_value(vc) * vs).to(torch.float32).transpose(2, 3).contiguous()
            same = orc.paged_attention_decode(q, kf, vf, tables, cl, scale)
            assert_close(got, same, 1e-15, "e4m3 decode vs fp32-cache decode")


def pin_append_e4m3_placement_and_values(orc: Oracle):
    """The 8-bit append changes exactly the addressed K rows and V columns
    (V pages are transposed); the codes are PyTorch's float8 cast of
    binary32(rope(k) / k_scale) and binary32(v / v_scale); q is rotated and
    rounded to its own type as in the plain append."""
    for dtype in (torch.bfloat16, torch.float32):
        q, k, v, pos, slots, NB, bs = _append_case(dtype, 43)
        T, Hq, d = q.shape
        Hkv = k.shape[1]
        ks, vs = 0.0173, 0.0291
        kc = torch.full((NB, Hkv, bs, d), 0x7F, dtype=torch.uint8)
        vc = torch.full((NB, Hkv, d, bs), 0x7F, dtype=torch.uint8)
        q2 = q.clone()
        orc.kv_append_e4m3(q2, k.clone(), v.clone(), pos, slots, kc, vc, 5e5, ks, vs)
        want_k = torch.zeros(NB, Hkv, bs, dtype=torch.bool)
        for s in slots.tolist():
            if s >= 0:
                want_k[s // bs, :, s % bs] = True
        kchg, vchg = kc != 0x7F, vc != 0x7F
        assert torch.equal(kchg.any(-1), want_k), "k rows written"
        assert torch.equal(vchg.any(-2), want_k), "v columns written"

        def rot(x, p):
            i = torch.arange(d // 2, dtype=torch.float64)
            z = torch.complex(x[..., : d // 2].double(), x[..., d // 2:].double())
            z = z * torch.exp(1j * float(p) * 5e5 ** (-2.0 * i / d))
            return torch.cat([z.real, z.imag], -1)

        def cast(x):
            return x.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)

        for t, s in enumerate(slots.tolist()):
            want_q = orc.round_bf16(rot(q[t], pos[t])) if dtype == torch.bfloat16 \
                else rot(q[t], pos[t]).to(torch.float32)
            assert (q2[t].double() - want_q.double()).abs().max().item() <= \
                (1e-6 if dtype == torch.float32 else 0.0), f"q token {t}"
            if s < 0:
                continue
            kk = rot(k[t], pos[t]) / ks
            got_k = kc[s // bs, :, s % bs]
            exact = cast(kk)
            # the rotation's last fp64 bit may differ from PyTorch's complex
            # product: allow a neighbouring code only where binary32(kk) sits
            # within a few binary32 ulps of an E4M3 midpoint
            near = torch.zeros_like(exact, dtype=torch.bool)
            for sgn in (-1, 1):
                nudged = kk.to(torch.float32)
                for _ in range(3):
                    nudged = torch.nextafter(nudged, torch.full_like(nudged, sgn * 1e9))
                near |= cast(nudged.double()) != exact
            assert bool(((got_k == exact) | near).all()), f"k codes token {t}"
            assert torch.equal(vc[s // bs, :, :, s % bs], cast(v[t].double() / vs)), f"v codes {t}"



def pin_sliding_window_decode(orc: Oracle):
    """A sliding window of W tokens equals attention over the last W tokens
    of the context (PyTorch fp64 SDPA on that slice), for bf16 and fp32
    storage, GQA groups and the 8-bit cache; a window at least as long as
    the context changes nothing; W = 1 returns the last token's V exactly
    ("Efficient LLM Inference", KV Caching: positions and windows)."""
    lens = [40, 17, 5, 33]
    cl = torch.tensor(lens, dtype=torch.int32)
    for dtype, Hq, Hkv in ((torch.float32, 8, 2), (torch.bfloat16, 4, 4)):
        kpool, vpool, tables, Ks, Vs = random_paged(lens, Hkv, 16, 16, dtype, 80)
        q = torch.randn(len(lens), Hq, 16, generator=_gen(81)).to(dtype)
        full = orc.paged_attention_decode(q, kpool, vpool, tables, cl, 0.25)
        for W in (1, 7, 16, 17, 33, 100):
            got = orc.paged_attention_decode(q, kpool, vpool, tables, cl, 0.25, window=W)
            for b, L in enumerate(lens):
                if W >= L:
                    assert torch.equal(got[b], full[b]), f"window {W} >= L {L} changed the result"
                    continue
                s0 = L - W
                want = sdpa(q[b][None].double(), Ks[b][s0:].double(), Vs[b][s0:].double(), 0.25)[0]
                assert_close(got[b], want, 1e-12, f"window {W} b={b}")
                if W == 1:
                    G = Hq // Hkv
                    last = Vs[b][L - 1].double().repeat_interleave(G, dim=0)
                    assert torch.equal(got[b], last), "W = 1 is not the last V"
    kc, vc, tables, Ks, Vs = _random_e4m3_cache(lens, 2, 16, 16, 82)
    q = torch.randn(len(lens), 8, 16, generator=_gen(83)).to(torch.bfloat16)
    got = orc.paged_attention_decode_e4m3(q, kc, vc, tables, cl, 0.25, 0.05, 0.07, window=9)
    for b, L in enumerate(lens):
        s0 = max(0, L - 9)
        want = sdpa(q[b][None].double(), _e4m3_value(Ks[b][s0:]) * 0.05,
                    _e4m3_value(Vs[b][s0:]) * 0.07, 0.25)[0]
        assert_close(got[b], want, 1e-12, f"e4m3 window b={b}")


def pin_sliding_window_chunked_prefill(orc: Oracle):
    """A windowed prefill chunk equals PyTorch's fp64 SDPA over the gathered
    context with a banded causal mask: query row r attends to keys
    r - W + 1 .. r."""
    for (Hq, Hkv, d, lens, C, W, seed) in [(8, 2, 16, [40, 17, 5], 5, 7, 84),
                                           (4, 4, 8, [33], 33, 16, 85)]:
        kpool, vpool, tables, Ks, Vs = random_paged(lens, Hkv, d, 16, torch.float32, seed)
        q = torch.randn(len(lens), C, Hq, d, generator=_gen(seed + 100))
        got = orc.paged_chunked_prefill(q, kpool, vpool, tables,
                                        torch.tensor(lens, dtype=torch.int32), 0.25, window=W)
        for b, L in enumerate(lens):
            G = Hq // Hkv
            Kr = Ks[b].double().repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
            Vr = Vs[b].double().repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
            Q = torch.zeros(L, Hq, d, dtype=torch.float64)
            Q[L - C:] = q[b].double()
            r = torch.arange(L)[:, None]
            t = torch.arange(L)[None, :]
            band = (t <= r) & (t > r - W)
            want = F.scaled_dot_product_attention(Q.permute(1, 0, 2)[None], Kr, Vr,
                                                  attn_mask=band, scale=0.25)[0].permute(1, 0, 2)
            assert_close(got[b], want[L - C:], 1e-12, f"windowed chunk b={b}")

PINS = [
    pin_round_bf16_matches_torch_cast,
    pin_round_bf16_single_rounding,
    pin_bf16_widening_exact,
    pin_rope_position_zero_is_identity,
    pin_rope_matches_hf_llama,
    pin_rope_is_complex_rotation,
    pin_decode_matches_sdpa,
    pin_decode_is_last_row_of_causal_prefill,
    pin_paged_equals_contiguous,
    pin_block_relabel_invariance,
    pin_closed_forms,
    pin_gqa_group_mapping,
    pin_empty_context,
    pin_exact_arithmetic_tiny,
    pin_append_placement_and_values,
    pin_append_rejects_out_of_range_slot,
    pin_append_then_decode_is_causal_last_row,
    pin_chunked_prefill_matches_causal_sdpa,
    pin_e4m3_decode_matches_torch,
    pin_e4m3_round_matches_torch_cast,
    pin_e4m3_quantizer_rounds_through_binary32,
    pin_e4m3_decode_matches_sdpa_over_dequantized,
    pin_append_e4m3_placement_and_values,
    pin_sliding_window_decode,
    pin_sliding_window_chunked_prefill,
]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.default)


# ---------------------------------------------------------------- planted mistakes
# Each entry: (name, exact text in pkv_oracle.c, replacement).  The mutated
# copy of the oracle is compiled on the CPU and must fail at least one pin.

MUTATIONS = [
    ("drop_scale", "s[t] = J->scale * acc;", "s[t] = acc;"),
    ("gqa_modulo", "const int64_t kvh = h / G;\n    const int64_t L = J->context_lens[b];",
     "const int64_t kvh = h % J->Hkv;\n    const int64_t L = J->context_lens[b];"),
    ("pool_head_major", "int64_t idx = ((blk * J->Hkv + kvh) * J->bs + row) * J->d + i;",
     "int64_t idx = ((kvh * J->num_blocks + blk) * J->bs + row) * J->d + i;"),
    ("row_index", "int64_t idx = ((blk * J->Hkv + kvh) * J->bs + row) * J->d + i;",
     "int64_t idx = ((blk * J->Hkv + kvh) * J->bs + (row + 1) % J->bs) * J->d + i;"),
    ("drop_last_token", "for (int64_t t = t0; t < L; ++t) {\n        double w",
     "for (int64_t t = t0; t + 1 < L; ++t) {\n        double w"),
    ("normalise_by_length", "for (int64_t i = 0; i < d; ++i) o[i] /= den;\n    return ORC_OK;",
     "for (int64_t i = 0; i < d; ++i) o[i] /= (double)L;\n    return ORC_OK;"),
    ("rope_sign", "x[i] = x0 * c - x1 * s;", "x[i] = x0 * c + x1 * s;"),
    ("rope_interleaved", "double x0 = x[i], x1 = x[i + half];\n        x[i] = x0 * c - x1 * s;\n        x[i + half] = x1 * c + x0 * s;",
     "if (2 * i + 1 >= d) continue;\n        double x0 = x[2 * i], x1 = x[2 * i + 1];\n        x[2 * i] = x0 * c - x1 * s;\n        x[2 * i + 1] = x1 * c + x0 * s;"),
    ("rope_frequency", "double freq = pow(theta, -(2.0 * (double)i) / (double)d);",
     "double freq = pow(theta, -((double)i) / (double)d);"),
    ("bf16_double_rounding", "double r = nearbyint(ldexp(a, -spacing_exp));",
     "double r = nearbyint(ldexp((double)(float)a, -spacing_exp));"),
    ("slot_offset", "int64_t blk = slot / bs, off = slot % bs;",
     "int64_t blk = slot / bs, off = (slot + 1) % bs;"),
    ("rotate_v", "/* v is copied unchanged, so its bits must survive exactly */",
     "for (int64_t i = 0; i < d; ++i) row[i] = load_elem(v_new, dtype, src + i);\n"
     "            rope_rotate(row, d, pos, theta);\n"
     "            for (int64_t i = 0; i < d; ++i) store_elem((void*)v_new, dtype, src + i, row[i]);"),
    ("e4m3_bias", "v = ldexp(1.0 + m / 8.0, E - 7);", "v = ldexp(1.0 + m / 8.0, E - 8);"),
    ("e4m3_subnormal", "v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    ("e4m3_spacing", "int spacing_exp = (e - 1) - 3;", "int spacing_exp = (e - 1) - 4;"),
    ("e4m3_no_saturation", "if (r > 448.0) r = 448.0;", ""),
    ("e4m3_no_binary32_step", "return double_to_e4m3((double)(float)(x / scale));",
     "return double_to_e4m3(x / scale);"),
    ("e4m3_scale_multiplies", "return double_to_e4m3((double)(float)(x / scale));",
     "return double_to_e4m3((double)(float)(x * scale));"),
    ("e4m3_v_row_major_store", "v_cache[page + i * bs + r] =", "v_cache[page + r * d + i] ="),
    ("e4m3_slot_offset", "int64_t blk = slot / bs, r = slot % bs;",
     "int64_t blk = slot / bs, r = (slot + 1) % bs;"),
    ("e4m3_v_row_major_load", "int64_t idx = ((blk * J->Hkv + kvh) * J->d + i) * J->bs + row;",
     "int64_t idx = ((blk * J->Hkv + kvh) * J->bs + row) * J->d + i;"),
    ("e4m3_drop_k_scale", "return e4m3_to_double(((const uint8_t*)J->k_cache)[idx]) * J->k_scale;",
     "return e4m3_to_double(((const uint8_t*)J->k_cache)[idx]);"),
    ("e4m3_drop_v_scale", "return e4m3_to_double(((const uint8_t*)J->v_cache)[idx]) * J->v_scale;",
     "return e4m3_to_double(((const uint8_t*)J->v_cache)[idx]);"),
    ("e4m3_k_unrotated", "for (int64_t i = 0; i < d; ++i) k_cache[page + r * d + i] =",
     "for (int64_t i = 0; i < d; ++i) row[i] = load_elem(k_new, dtype, src + i);\n"
     "            for (int64_t i = 0; i < d; ++i) k_cache[page + r * d + i] ="),
    ("window_start_late", "const int64_t t0 = (J->window > 0 && L > J->window) ? L - J->window : 0;",
     "const int64_t t0 = (J->window > 0 && L > J->window) ? L - J->window + 1 : 0;"),
    ("window_start_early", "const int64_t t0 = (J->window > 0 && L > J->window) ? L - J->window : 0;",
     "const int64_t t0 = (J->window > 0 && L > J->window) ? L - J->window - 1 : 0;"),
    ("skip_q_rotation", "rope_rotate(row, d, pos, theta);\n        for (int64_t i = 0; i < d; ++i) store_elem(q,",
     "for (int64_t i = 0; i < d; ++i) store_elem(q,"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new, tmp_path):
    src = open(oracle_build.SRC).read()
    assert src.count(old) == 1, f"mutation {name} does not match the oracle source exactly once"
    mutant_src = tmp_path / f"mut_{name}.c"
    mutant_src.write_text(src.replace(old, new))
    lib = oracle_build.compile_source(str(mutant_src), str(tmp_path / f"libmut_{name}.so"))
    mutant = Oracle(lib)
    caught = []
    for pin in PINS:
        try:
            pin(mutant)
        except (AssertionError, OracleError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"


# Planted mistakes in the oracle's Python layer (argument marshalling and the
# chunked prefill built on the decode): the mutated copy of oracle/__init__.py
# is loaded as its own module over the unmodified C library.
PY_MUTATIONS = [
    ("prefill_query_misses_own_token",
     "lens_i = (context_lens.to(torch.int64) - C + i + 1).clamp(min=0)",
     "lens_i = (context_lens.to(torch.int64) - C + i).clamp(min=0)"),
    ("prefill_not_causal_in_chunk",
     "lens_i = (context_lens.to(torch.int64) - C + i + 1).clamp(min=0)",
     "lens_i = context_lens.to(torch.int64).clamp(min=0)"),
    ("prefill_ignores_window",
     "nthreads=nthreads, window=window)\n        return out\n\n    def contiguous_decode",
     "nthreads=nthreads, window=0)\n        return out\n\n    def contiguous_decode"),
    ("e4m3_scales_swapped",
     "float(scale), float(k_scale), float(v_scale),\n                                              int(window)",
     "float(scale), float(v_scale), float(k_scale),\n                                              int(window)"),
    ("e4m3_append_scales_swapped",
     "T, Hq, Hkv, d, NB, bs, float(rope_theta),\n                                           float(k_scale), float(v_scale))",
     "T, Hq, Hkv, d, NB, bs, float(rope_theta),\n                                           float(v_scale), float(k_scale))"),
    ("decode_window_dropped",
     "float(scale), int(window), pp, npairs, int(nthreads),",
     "float(scale), 0, pp, npairs, int(nthreads),"),
]


def _oracle_module_copy(name, src):
    import types

    mod = types.ModuleType(f"oracle._copy_{name}")
    mod.__package__ = "oracle"
    mod.__file__ = oracle.__file__
    exec(compile(src, f"<oracle copy {name}>", "exec"), mod.__dict__)
    # the copy raises the original error class, which the pins expect
    mod.OracleError = OracleError
    return mod


def test_unmutated_module_copy_passes_every_pin():
    """Control for the harness below: loading the module this way changes
    nothing by itself."""
    copy = _oracle_module_copy("control", open(oracle.__file__).read()).Oracle()
    for pin in PINS:
        pin(copy)


@pytest.mark.parametrize("name,old,new", PY_MUTATIONS, ids=[m[0] for m in PY_MUTATIONS])
def test_planted_marshalling_mistake_is_caught(name, old, new):
    src = open(oracle.__file__).read()
    assert src.count(old) == 1, f"mutation {name} does not match the oracle module exactly once"
    mutant = _oracle_module_copy(name, src.replace(old, new)).Oracle()
    caught = []
    for pin in PINS:
        try:
            pin(mutant)
        except (AssertionError, OracleError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
