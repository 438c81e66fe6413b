// paged_prefill.cu -- multi-query (chunked-prefill) attention over a paged KV
// cache on sm_100a.
//
// What it computes ("Efficient LLM Inference", KV Caching: chunked computation
// over the retained K/V equals the full-prefix pass; "Inference From Scratch",
// ch. 10 paged attention and ch. 8 online softmax): every sequence b has a
// chunk of C query tokens, the last C tokens of its context (their K/V
// already appended to the cache).  Query i sits at position L_b - C + i and
// attends causally to tokens 0 .. L_b - C + i:
//   out[b, i, h, :] = softmax_t(scale q[b, i, h] . K_b[t]) V_b[t],  t <= L_b - C + i,
// with kv head h / G.  That is the decode definition applied to each query
// with its own context length, which is how the tests check it.
//
// Work decomposition.  A work item is (sequence, kv head, row group,
// partition of P keys).  Its rows are up to 32 (query, head) pairs of the kv
// head, (query i, head g) -> row i*G + g; each of the four consumer warps
// owns 8 rows and runs them over every page of the partition, so a K/V page
// is read once per row group.  One CTA per item (no persistence: the items
// of a prefill chunk are uniform).  Partitions are merged by a log-sum-exp
// combine kernel when a sequence has more than one.
//
// Inside a CTA: one producer warp turns block-table entries into TMA loads of
// whole K and V pages (128-byte swizzle) into a ring of stages guarded by
// mbarriers; the consumer warps compute S = Q K^T and O += P V with
// mma.sync m16n8k16 (bf16 in, fp32 accumulate).  A warp's 16-row A tile
// holds its 8 rows twice: rows r carry the high bf16 part of P, rows r + 8
// the low part (p = hi + lo to ~2^-17 relative).  Each row masks the keys
// past its own position; a row can have no key in a page or a partition
// (its softmax state then stays m = -inf, l = 0).  Every wait is bounded.
#include <cuda_bf16.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

using bf16 = __nv_bfloat16;
constexpr int NWP = 4;                        // consumer warps
constexpr int kRowsPerWarp = 8;               // (query, head) rows per warp
constexpr int kThreadsP = (NWP + 1) * 32;     // + one producer warp
constexpr float kNegInfP = -__builtin_huge_valf();

template <int D>
struct PLayout {
    static constexpr int PAGE_BYTES = kPageRows * D * 2;
    static constexpr int BOXES = D / 64;            // 64-column TMA boxes per page
    static constexpr int BOX_BYTES = PAGE_BYTES / BOXES;
    static constexpr int SP = 4;                    // pages per stage
    static constexpr int STAGE_BYTES = 2 * SP * PAGE_BYTES;  // SP K pages, then SP V pages
    static constexpr int STAGES = D == 64 ? 4 : 3;  // 64 KiB / 96 KiB of ring
    static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
    static constexpr int OFF_MASK = OFF_BAR + 2 * STAGES * 8;  // full, empty
    static constexpr size_t SMEM = 1024 + OFF_MASK + STAGES * 4 + 16;
};

struct PrefillParams {
    const bf16* q;              // [B, C, Hq, D]
    const int32_t* block_tables;
    const int32_t* context_lens;
    void* out;                  // [B, C, Hq, D]
    float* part_o;              // [B, C, Hq, NP, D]
    float* part_ml;             // [B, C, Hq, NP, 2]
    int32_t* err;
    int B, C, Hq, Hkv, MB, P, NP, RG, num_blocks;
    float scale_log2;
    int out_bf16;
    int window;                 // sliding window: query at position t sees t - window + 1 .. t
};

// Byte offset of 16-byte chunk c of token row tok in a 128-byte-swizzled page.
template <int D>
__device__ __forceinline__ uint32_t pchunk(int tok, int c) {
    if constexpr (D == 64) {
        return tok * 128 + ((c ^ (tok & 7)) << 4);
    } else {
        return (c >> 3) * 2048 + tok * 128 + (((c & 7) ^ (tok & 7)) << 4);
    }
}

__device__ __forceinline__ void pstore(void* out, size_t idx, float v, int out_bf16) {
    if (out_bf16)
        reinterpret_cast<bf16*>(out)[idx] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float*>(out)[idx] = v;
}

// The item's sequence and key range, from blockIdx.x.
struct PItem {
    int b, h, rg, part, L, np, t0, t1, npages;
    int lo;  // sliding window: first token any query of the chunk attends (0 otherwise)
};

__device__ __forceinline__ PItem prefill_item(const PrefillParams& p) {
    PItem it;
    int x = blockIdx.x;
    it.part = x % p.NP;
    x /= p.NP;
    it.rg = x % p.RG;
    x /= p.RG;
    it.h = x % p.Hkv;
    it.b = x / p.Hkv;
    int L = p.context_lens[it.b];
    const int maxlen = p.MB * kPageRows;
    if (L < p.C || L > maxlen) {
        // the chunk must lie inside the context
        if (it.part == 0 && it.rg == 0 && it.h == 0 && threadIdx.x == 0)
            report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
        L = L < p.C ? 0 : maxlen;
    }
    it.L = L;
    it.np = (L + p.P - 1) / p.P;
    // sliding window: pages before the chunk's first query's window are not
    // read (a partition wholly before it has no pages and leaves an empty
    // partial)
    it.lo = (p.window > 0 && L - p.C + 1 > p.window) ? L - p.C + 1 - p.window : 0;
    it.t0 = max(it.part * p.P, it.lo / kPageRows * kPageRows);
    it.t1 = min(L, it.part * p.P + p.P);
    it.npages = it.t1 > it.t0 ? (it.t1 - it.t0 + kPageRows - 1) / kPageRows : 0;
    return it;
}

template <int D>
__device__ void prefill_producer(const PrefillParams& p, const PItem& it, const CUtensorMap* tmk,
                                 const CUtensorMap* tmv, uint8_t* base, uint64_t* full,
                                 uint64_t* empty, uint32_t* masks, volatile int* s_abort) {
    using L = PLayout<D>;
    const int lane = threadIdx.x & 31;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_parity[8];
    uint32_t issued_any = 0;
    bool abort = false;
    // block-table entries of the next 32-page chunk are loaded while this one
    // is issued, and range-checked when their chunk comes up
    const int32_t* row_tab = p.block_tables + (size_t)it.b * p.MB + it.t0 / kPageRows;
    int raw = lane < it.npages ? row_tab[lane] : -1;
    for (int c0 = 0; c0 < it.npages && !abort; c0 += 32) {
        int ent = -1;
        if (c0 + lane < it.npages) {
            if (raw < 0 || raw >= p.num_blocks)
                report_error(p.err, PKV_DEVERR_BLOCK_ID);
            else
                ent = raw;
        }
        raw = c0 + 32 + lane < it.npages ? row_tab[c0 + 32 + lane] : -1;
        const int cend = min(it.npages, c0 + 32);
        for (int s0 = c0; s0 < cend; s0 += L::SP) {
            const int npg = min(L::SP, it.npages - s0);
            const int k = lane - (s0 - c0);
            const bool mine = k >= 0 && k < npg && ent >= 0;
            const uint32_t vmask = __ballot_sync(0xffffffffu, mine) >> (s0 - c0);
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1) && !*s_abort;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                abort = true;
                break;
            }
            if (lane == 0) {
                masks[stage] = vmask;
                mbar_arrive_expect_tx(&full[stage], __popc(vmask) * 2u * L::PAGE_BYTES);
            }
            __syncwarp();
            if (mine) {
                uint8_t* kdst = base + stage * L::STAGE_BYTES + k * L::PAGE_BYTES;
                uint8_t* vdst = kdst + L::SP * L::PAGE_BYTES;
                const int row0 = (ent * p.Hkv + it.h) * kPageRows;
#pragma unroll
                for (int bx = 0; bx < L::BOXES; ++bx) {
                    tma_load_2d(kdst + bx * L::BOX_BYTES, tmk, bx * 64, row0, &full[stage]);
                    tma_load_2d(vdst + bx * L::BOX_BYTES, tmv, bx * 64, row0, &full[stage]);
                }
            }
            issued_parity[stage] = phase;
            issued_any |= 1u << stage;
            if (++stage == L::STAGES) {
                stage = 0;
                phase ^= 1;
            }
        }
    }
    if (abort) {
        *s_abort = 1;
        if (lane == 0) {
            report_error(p.err, PKV_DEVERR_TIMEOUT);
            for (int s = 0; s < L::STAGES; ++s)
                if (issued_any & (1u << s)) (void)mbar_wait(&full[s], issued_parity[s]);
        }
        __syncwarp();
    }
}

// One query row of a consumer lane (lanes 4r .. 4r+3 of a warp share row r).
struct PRow {
    bool ok;            // the row exists
    const bf16* q;      // its query vector (D elements)
    int len;            // it may attend to tokens t < len
    int lo;             // and t >= lo (sliding window; 0 otherwise)
    bool direct;        // write the output row (else a partition partial)
    void* out;          // direct: the output row (D elements of out_bf16 ? bf16 : f32)
    float* po;          // partial: o (D floats)
    float* pml;         // partial: (m, l)
};

// A consumer warp runs its 8 rows over every page of the item's key range
// [t0, t1): S = Q K^T and O += P V on the tensor cores, online softmax per
// row in the log2 domain, keys at t >= row.len masked per row.
template <int D>
__device__ void multirow_consumer(float scale_log2, int out_bf16, int32_t* err, const PItem& it,
                                  const PRow& row, uint8_t* base, uint64_t* full, uint64_t* empty,
                                  const uint32_t* masks, volatile int* s_abort) {
    using L = PLayout<D>;
    constexpr int KS = D / 16, NT = D / 8;
    const int lane = threadIdx.x & 31;
    const int cq = lane & 3;
    const bool row_ok = row.ok;
    const int row_len = row_ok ? row.len : 0;
    const int row_lo = row.lo;

    // A fragments of Q: rows r and r + 8 both hold this lane's row
    uint32_t qa[KS][2];
    {
        const uint32_t* qr = reinterpret_cast<const uint32_t*>(row.q);
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            const int col = kk * 16 + 2 * cq;
            qa[kk][0] = row_ok ? qr[col / 2] : 0u;
            qa[kk][1] = row_ok ? qr[(col + 8) / 2] : 0u;
        }
    }
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_run = kNegInfP, l_run = 0.f;

    int stage = 0;
    uint32_t phase = 0;
    const int mi = lane >> 3, ri = lane & 7;
    const int nst = (it.npages + L::SP - 1) / L::SP;
    bool ok = true;
    for (int s = 0; s < nst; ++s) {
        ok = mbar_wait(&full[stage], phase) && !*s_abort;
        if (!ok) break;
        const uint32_t msk = masks[stage];
        for (int u = 0; u < L::SP; ++u) {
            const int j = s * L::SP + u;
            if (j >= it.npages || !((msk >> u) & 1u)) continue;
            const int tbase = it.t0 + j * kPageRows;       // absolute token of page row 0
            const int in_part = min(kPageRows, it.t1 - tbase);   // rows inside the partition
            const int row_valid = max(0, min(in_part, row_len - tbase));
            const int row_first = max(0, row_lo - tbase);   // sliding window
            const uint32_t kbase = smem_addr(base + stage * L::STAGE_BYTES + u * L::PAGE_BYTES);
            const uint32_t vbase = kbase + L::SP * L::PAGE_BYTES;
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int tok = ri + ((mi >> 1) << 3);
                const int ch = 2 * kk + (mi & 1);
                uint32_t b00, b01, b10, b11;
                ldsm_x4(kbase + pchunk<D>(tok, ch), b00, b01, b10, b11);
                const uint32_t a[4] = {qa[kk][0], qa[kk][0], qa[kk][1], qa[kk][1]};
                mma_bf16_16816(sc[0], a, b00, b01);
                mma_bf16_16816(sc[1], a, b10, b11);
            }
            float x[2][2];
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tk = n * 8 + 2 * cq + e;
                    x[n][e] = (tk < row_valid && tk >= row_first) ? sc[n][e] * scale_log2
                                                                  : kNegInfP;
                }
            float mx = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run, mx);
            // a row with no key so far keeps m = -inf: use 0 as the reference
            const float m_ref = m_new == kNegInfP ? 0.f : m_new;
            const float alpha = fast_exp2(m_run - m_ref);
            float pr[2][2];
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e) pr[n][e] = fast_exp2(x[n][e] - m_ref);
            l_run = l_run * alpha + ((pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
            if (__any_sync(0xffffffffu, m_new != m_run)) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    o[n][0] *= alpha;
                    o[n][1] *= alpha;
                    o[n][2] *= alpha;
                    o[n][3] *= alpha;
                }
            }
            m_run = m_new;
            // P: rows r the high bf16 part, rows r + 8 the low part
            uint32_t pa[4];
            {
                const uint32_t hi0 = pack_bf16(pr[0][0], pr[0][1]);
                const uint32_t hi1 = pack_bf16(pr[1][0], pr[1][1]);
                pa[0] = hi0;
                pa[1] = pack_bf16(pr[0][0] - bf16lo(hi0), pr[0][1] - bf16hi(hi0));
                pa[2] = hi1;
                pa[3] = pack_bf16(pr[1][0] - bf16lo(hi1), pr[1][1] - bf16hi(hi1));
            }
            // V rows past the partition may hold stale shared memory, and rows
            // before every query's window are not attended: zero them
            uint32_t vmask_lo = 0xffffffffu, vmask_hi = 0xffffffffu;
            const int v_first = max(0, it.lo - tbase);
            if (in_part < kPageRows || v_first > 0) {
                const int k0 = 2 * cq;
                auto in = [&](int k) { return k >= v_first && k < in_part; };
                vmask_lo = (in(k0) ? 0x0000ffffu : 0u) | (in(k0 + 1) ? 0xffff0000u : 0u);
                vmask_hi = (in(k0 + 8) ? 0x0000ffffu : 0u) | (in(k0 + 9) ? 0xffff0000u : 0u);
            }
#pragma unroll
            for (int c = 0; c < NT; c += 2) {
                const int tok = ri + ((mi & 1) << 3);
                const int ch = c + (mi >> 1);
                uint32_t v0, v1, v2, v3;
                ldsm_x4_trans(vbase + pchunk<D>(tok, ch), v0, v1, v2, v3);
                mma_bf16_16816(o[c], pa, v0 & vmask_lo, v1 & vmask_hi);
                mma_bf16_16816(o[c + 1], pa, v2 & vmask_lo, v3 & vmask_hi);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1;
        }
    }
    if (!ok) {
        *s_abort = 1;
        if (lane == 0) report_error(err, PKV_DEVERR_TIMEOUT);
        return;
    }
    // row result: high + low rows, row sum over the quad
    float lsum = l_run;
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    if (!row_ok) return;
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    if (row.direct) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int col = n * 8 + 2 * cq;
            pstore(row.out, col, (o[n][0] + o[n][2]) * inv, out_bf16);
            pstore(row.out, col + 1, (o[n][1] + o[n][3]) * inv, out_bf16);
        }
    } else {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int col = n * 8 + 2 * cq;
            *reinterpret_cast<float2*>(row.po + col) =
                make_float2((o[n][0] + o[n][2]) * inv, (o[n][1] + o[n][3]) * inv);
        }
        if (cq == 0) {
            row.pml[0] = m_run;
            row.pml[1] = lsum;
        }
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kThreadsP)
    paged_prefill_kernel(const __grid_constant__ PrefillParams p,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v) {
    using L = PLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L::OFF_BAR);
    uint64_t* empty = full + L::STAGES;
    uint32_t* masks = reinterpret_cast<uint32_t*>(base + L::OFF_MASK);
    volatile int* s_abort = reinterpret_cast<volatile int*>(masks + L::STAGES);
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NWP);
        }
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == NWP && (tid & 31) == 0) {
        prefetch_tensor_map(&tm_k);
        prefetch_tensor_map(&tm_v);
    }
    grid_dependency_wait();
    grid_launch_dependents();
    const PItem it = prefill_item(p);
    __syncthreads();
    if (it.part >= it.np) return;  // no keys in this partition (whole CTA leaves)
    if (warp == NWP) {
        prefill_producer<D>(p, it, &tm_k, &tm_v, base, full, empty, masks, s_abort);
        return;
    }
    // this lane's row: (query i, head g) of the item's row group; query i
    // sees tokens 0 .. L - C + i
    PRow row;
    const int fr = it.rg * (NWP * kRowsPerWarp) + warp * kRowsPerWarp + ((tid & 31) >> 2);
    row.ok = fr < p.C * G;
    const int qi = row.ok ? fr / G : 0, hq = it.h * G + (row.ok ? fr % G : 0);
    const size_t r = ((size_t)it.b * p.C + qi) * p.Hq + hq;
    row.q = p.q + r * D;
    row.len = it.L - p.C + qi + 1;
    row.lo = (p.window > 0 && row.len > p.window) ? row.len - p.window : 0;
    row.direct = it.np == 1;
    row.out = p.out_bf16 ? (void*)(reinterpret_cast<bf16*>(p.out) + r * D)
                         : (void*)(reinterpret_cast<float*>(p.out) + r * D);
    row.po = p.part_o ? p.part_o + (r * p.NP + it.part) * D : nullptr;
    row.pml = p.part_ml ? p.part_ml + (r * p.NP + it.part) * 2 : nullptr;
    multirow_consumer<D>(p.scale_log2, p.out_bf16, p.err, it, row, base, full, empty, masks,
                         s_abort);
}

// out[b, i, h, :] from the partials of the sequence's partitions (the same
// log-sum-exp merge as the decode's combine).  One warp per (b, i, h).
template <int D>
__global__ void __launch_bounds__(128) prefill_combine_kernel(const __grid_constant__ PrefillParams p) {
    grid_dependency_wait();
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);  // (b * C + i) * Hq + h
    if (row >= (int64_t)p.B * p.C * p.Hq) return;
    const int b = (int)(row / ((int64_t)p.C * p.Hq));
    int L = p.context_lens[b];
    const int maxlen = p.MB * kPageRows;
    L = L < p.C ? 0 : (L > maxlen ? maxlen : L);
    const int np = (L + p.P - 1) / p.P;
    if (np <= 1) return;  // written by the attention kernel
    const float* ml = p.part_ml + row * p.NP * 2;
    float M = kNegInfP;
    for (int k = lane; k < np; k += 32) M = fmaxf(M, ml[2 * k]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    constexpr int PER = D / 32;
    float acc[PER], den = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    for (int k = 0; k < np; ++k) {
        const float m = ml[2 * k], l = ml[2 * k + 1];
        const float w = (m == kNegInfP || l == 0.f) ? 0.f : l * fast_exp2(m - M);
        den += w;
        const float* po = p.part_o + (row * p.NP + k) * D;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = fmaf(w, po[lane + 32 * e], acc[e]);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) pstore(p.out, row * D + lane + 32 * e, acc[e] * inv, p.out_bf16);
}

// ---- cascade decode: the shared-prefix pass ----------------------------------

struct CascadeParams {
    const bf16* q;                  // [B, Hq, D], rotated (kv_append ran before)
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* group_start;     // [NG + 1]: group g = sequences [gs[g], gs[g + 1])
    const int32_t* shared_tokens;   // [B]
    float* part_o;                  // decode workspace partials: NPT slots per (b, q head)
    float* part_ml;
    int32_t* err;
    int B, Hq, Hkv, MB, NPT, RG, NG, num_blocks;
    float scale_log2;
};

// Shared tokens of sequence b as the decode counts them: whole pages inside
// its (clamped) context.
__device__ __forceinline__ int cascade_shared(const CascadeParams& p, int b) {
    int L = p.context_lens[b];
    const int maxlen = p.MB * kPageRows;
    L = L < 0 ? 0 : (L > maxlen ? maxlen : L);
    int s = p.shared_tokens[b];
    return s < 0 ? 0 : (s > L ? L : s) / kPageRows * kPageRows;
}

// One CTA per (group, kv head, row group): the rows are (member, head)
// pairs, member m of the group and head g -> row m*G + g; every row attends
// to the first shared_tokens of its own sequence, read once for the group
// from the pages of the member that shares the most (the others' shared
// block-table entries must be the same ids: a mismatch sets
// PKV_DEVERR_PREFIX).  The result goes to partial slot 0 of each member;
// the decode kernel writes the rest of the sequence to slots 1.. and the
// combine merges them.  The kernel does not wait for the decode kernel before
// it starts (it reads nothing the decode writes), so its CTAs fill SMs as the
// decode's CTAs finish; each CTA waits for the decode grid before it exits,
// so that the combine, which waits for this grid, also sees the decode's
// partials.
template <int D, int G>
__global__ void __launch_bounds__(kThreadsP)
    cascade_prefix_kernel(const __grid_constant__ CascadeParams p,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v) {
    using L = PLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L::OFF_BAR);
    uint64_t* empty = full + L::STAGES;
    uint32_t* masks = reinterpret_cast<uint32_t*>(base + L::OFF_MASK);
    volatile int* s_abort = reinterpret_cast<volatile int*>(masks + L::STAGES);
    __shared__ int s_grp[3];  // first member, member count, leader
    __shared__ int s_len;     // the leader's shared tokens
    const int tid = threadIdx.x, warp = tid >> 5;
    grid_launch_dependents();
    int x = blockIdx.x;
    const int rg = x % p.RG;
    x /= p.RG;
    const int h = x % p.Hkv, g = x / p.Hkv;
    if (tid == 0) {
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NWP);
        }
        *s_abort = 0;
        fence_barrier_init();
        int gs = p.group_start[g], ge = p.group_start[g + 1];
        if (gs < 0 || ge < gs || ge > p.B) {
            report_error(p.err, PKV_DEVERR_PREFIX);
            gs = ge = 0;
        }
        int best = 0, leader = gs;
        for (int b = gs; b < ge; ++b) {
            const int sb = cascade_shared(p, b);
            if (sb > best) {
                best = sb;
                leader = b;
            }
        }
        s_grp[0] = gs;
        s_grp[1] = ge - gs;
        s_grp[2] = leader;
        s_len = best;
    }
    __syncthreads();
    const int gs = s_grp[0], nmem = s_grp[1], leader = s_grp[2], S = s_len;
    if (S > 0) {
        if (warp == NWP && (tid & 31) == 0) {
            prefetch_tensor_map(&tm_k);
            prefetch_tensor_map(&tm_v);
        }
        // every member's shared pages must be the leader's (checked once, by row group 0)
        if (rg == 0 && h == 0) {
            for (int idx = tid; idx < nmem * (S / kPageRows); idx += kThreadsP) {
                const int m = idx / (S / kPageRows), j = idx - m * (S / kPageRows);
                const int b = gs + m;
                if (j < cascade_shared(p, b) / kPageRows &&
                    p.block_tables[(size_t)b * p.MB + j] != p.block_tables[(size_t)leader * p.MB + j])
                    report_error(p.err, PKV_DEVERR_PREFIX);
            }
        }
        PItem it;
        it.b = leader;
        it.h = h;
        it.rg = rg;
        it.part = 0;
        it.L = S;
        it.np = 1;
        it.t0 = 0;
        it.t1 = S;
        it.npages = S / kPageRows;
        it.lo = 0;
        PrefillParams pp;  // the fields the page producer reads
        pp.block_tables = p.block_tables;
        pp.err = p.err;
        pp.MB = p.MB;
        pp.Hkv = p.Hkv;
        pp.num_blocks = p.num_blocks;
        if (warp == NWP) {
            prefill_producer<D>(pp, it, &tm_k, &tm_v, base, full, empty, masks, s_abort);
        } else {
            PRow row;
            const int fr = rg * (NWP * kRowsPerWarp) + warp * kRowsPerWarp + ((tid & 31) >> 2);
            const int m = fr / G, hq = h * G + fr % G;
            const int b = gs + m;
            row.ok = m < nmem;
            row.len = row.ok ? cascade_shared(p, b) : 0;
            row.lo = 0;
            row.ok = row.ok && row.len > 0;  // no shared tokens: no slot 0
            const size_t r = (size_t)(row.ok ? b : 0) * p.Hq + hq;
            row.q = p.q + r * D;
            row.direct = false;
            row.out = nullptr;
            row.po = p.part_o + (r * p.NPT) * D;
            row.pml = p.part_ml + (r * p.NPT) * 2;
            multirow_consumer<D>(p.scale_log2, 0, p.err, it, row, base, full, empty, masks,
                                 s_abort);
        }
    }
    // do not complete before the decode grid: the combine waits for this one
    if ((tid & 31) == 0) grid_dependency_wait();
}

int current_device_p() {
    int dev = 0;
    cudaGetDevice(&dev);
    return dev;
}

template <typename K>
cudaError_t set_smem_once(K kern, size_t smem) {
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, size_t> done;
    const auto key = std::make_pair(reinterpret_cast<const void*>(kern), current_device_p());
    std::lock_guard<std::mutex> lock(mu);
    auto f = done.find(key);
    if (f != done.end() && f->second >= smem) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) done[key] = smem;
    return e;
}

template <int D, int G>
cudaError_t launch_prefill_typed(const PrefillArgs& a, const CUtensorMap& tmk,
                                 const CUtensorMap& tmv) {
    using L = PLayout<D>;
    auto kern = paged_prefill_kernel<D, G>;
    cudaError_t e = set_smem_once(kern, L::SMEM);
    if (e != cudaSuccess) return e;
    PrefillParams p;
    p.q = static_cast<const bf16*>(a.q);
    p.block_tables = a.block_tables;
    p.context_lens = a.context_lens;
    p.out = a.out;
    p.part_o = a.part_o;
    p.part_ml = a.part_ml;
    p.err = a.device_error;
    p.B = (int)a.B;
    p.C = (int)a.C;
    p.Hq = (int)a.Hq;
    p.Hkv = (int)a.Hkv;
    p.MB = (int)a.MB;
    p.P = a.partition_tokens;
    p.NP = a.max_partitions;
    p.RG = (int)((a.C * G + NWP * kRowsPerWarp - 1) / (NWP * kRowsPerWarp));
    p.num_blocks = (int)a.num_blocks;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out_bf16 = a.out_dtype == PKV_DTYPE_BF16;
    p.window = a.window;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.Hkv * p.RG * a.max_partitions));
    cfg.blockDim = dim3(kThreadsP);
    cfg.dynamicSmemBytes = L::SMEM;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, p, tmk, tmv);
    if (e != cudaSuccess || a.max_partitions <= 1) return e;

    cudaLaunchConfig_t cc = cfg;
    const int64_t rows = a.B * a.C * a.Hq;
    cc.gridDim = dim3((unsigned)((rows + 3) / 4));
    cc.blockDim = dim3(128);
    cc.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cc, prefill_combine_kernel<D>, p);
}

template <int D>
cudaError_t prefill_dispatch_g(const PrefillArgs& a, const CUtensorMap& k, const CUtensorMap& v) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_prefill_typed<D, 1>(a, k, v);
        case 2: return launch_prefill_typed<D, 2>(a, k, v);
        case 4: return launch_prefill_typed<D, 4>(a, k, v);
        case 8: return launch_prefill_typed<D, 8>(a, k, v);
    }
    return cudaErrorInvalidValue;
}

template <int D, int G>
cudaError_t launch_cascade_typed(const CascadeArgs& a, const CUtensorMap& tmk,
                                 const CUtensorMap& tmv) {
    using L = PLayout<D>;
    auto kern = cascade_prefix_kernel<D, G>;
    cudaError_t e = set_smem_once(kern, L::SMEM);
    if (e != cudaSuccess) return e;
    CascadeParams p;
    p.q = static_cast<const bf16*>(a.q);
    p.block_tables = a.block_tables;
    p.context_lens = a.context_lens;
    p.group_start = a.group_start;
    p.shared_tokens = a.shared_tokens;
    p.part_o = a.part_o;
    p.part_ml = a.part_ml;
    p.err = a.device_error;
    p.B = (int)a.B;
    p.Hq = (int)a.Hq;
    p.Hkv = (int)a.Hkv;
    p.MB = (int)a.MB;
    p.NPT = a.slots_per_row;
    p.RG = (int)((a.max_group_size * G + NWP * kRowsPerWarp - 1) / (NWP * kRowsPerWarp));
    p.NG = (int)a.num_groups;
    p.num_blocks = (int)a.num_blocks;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.num_groups * a.Hkv * p.RG));
    cfg.blockDim = dim3(kThreadsP);
    cfg.dynamicSmemBytes = L::SMEM;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p, tmk, tmv);
}

template <int D>
cudaError_t cascade_dispatch_g(const CascadeArgs& a, const CUtensorMap& k, const CUtensorMap& v) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_cascade_typed<D, 1>(a, k, v);
        case 2: return launch_cascade_typed<D, 2>(a, k, v);
        case 4: return launch_cascade_typed<D, 4>(a, k, v);
        case 8: return launch_cascade_typed<D, 8>(a, k, v);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_cascade_prefix(const CascadeArgs& a) {
    if (a.num_groups <= 0) return cudaSuccess;
    CUtensorMap tmk, tmv;
    cudaError_t e = encode_cache_map(&tmk, a.k_cache, a.num_blocks, a.Hkv, a.D, PKV_DTYPE_BF16);
    if (e != cudaSuccess) return e;
    e = encode_cache_map(&tmv, a.v_cache, a.num_blocks, a.Hkv, a.D, PKV_DTYPE_BF16);
    if (e != cudaSuccess) return e;
    return a.D == 64 ? cascade_dispatch_g<64>(a, tmk, tmv) : cascade_dispatch_g<128>(a, tmk, tmv);
}

cudaError_t launch_paged_prefill(const PrefillArgs& a) {
    CUtensorMap tmk, tmv;
    cudaError_t e = encode_cache_map(&tmk, a.k_cache, a.num_blocks, a.Hkv, a.D, PKV_DTYPE_BF16);
    if (e != cudaSuccess) return e;
    e = encode_cache_map(&tmv, a.v_cache, a.num_blocks, a.Hkv, a.D, PKV_DTYPE_BF16);
    if (e != cudaSuccess) return e;
    return a.D == 64 ? prefill_dispatch_g<64>(a, tmk, tmv) : prefill_dispatch_g<128>(a, tmk, tmv);
}

}  // namespace pkv
