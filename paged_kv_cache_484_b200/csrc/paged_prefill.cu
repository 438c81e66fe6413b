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
// partition of P keys).  Its rows are up to 128 (query, head) pairs of the kv
// head, (query i, head g) -> row i*G + g, one tile of a 5th-generation
// tensor-core MMA, so a K/V page is read once per row group.  One CTA per
// item, one CTA per SM.  Partitions are merged by a log-sum-exp combine kernel
// when a sequence has more than one.  The cascade decode's shared-prefix pass
// (the end of this file) runs its items through the same tile routine.
//
// Inside a CTA (umma_attend): one producer warp turns block-table entries
// into TMA loads of whole K and V pages (128-byte swizzle) into a ring of
// 64-key stages guarded by mbarriers; one lane issues tcgen05 MMAs, S = Q K^T
// and O += P V, with the accumulators in tensor memory; two softmax
// warpgroups (one thread per row each) take alternate tiles.  P is split
// into a high and a low bf16 part (p = hi + lo to ~2^-17 relative).  Each row
// masks the keys past its own position; a row can have no key in a tile or a
// partition (its softmax state then stays m = -inf, l = 0).  Every wait is
// bounded.
#include <cuda_bf16.h>

#include <algorithm>
#include <climits>
#include <map>
#include <mutex>
#include <tuple>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

using bf16 = __nv_bfloat16;
constexpr float kNegInfP = -__builtin_huge_valf();

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

// order: the sequences longest first (null: in order).
__device__ __forceinline__ PItem prefill_item(const PrefillParams& p, const int* order) {
    PItem it;
    int x = blockIdx.x;
    it.part = x % p.NP;
    x /= p.NP;
    it.rg = x % p.RG;
    x /= p.RG;
    it.h = x % p.Hkv;
    it.b = order ? order[x / p.Hkv] : x / p.Hkv;
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

// ---- attention tiles on the 5th-generation tensor cores ----------------------
//
// The chunked prefill (and the cascade's shared-prefix pass) run their items
// through one routine, umma_attend: an item is up to 128 rows -- (query,
// head) pairs of one kv head, the M of a tcgen05 MMA -- over a key range of
// one sequence's pages, so a K/V page is read once per 128 rows.  Both
// contractions run on the tensor cores with their accumulators in tensor
// memory:
//   S = Q K^T      (M = 128 rows, N = 64 keys, K = D), fp32
//   O += P V       (M = 128 rows, N = D, K = 64 keys), fp32
// P is split into a high and a low bf16 part (p = hi + lo to ~2^-17
// relative) and both are multiplied into O, as on the warp-level path.  The
// softmax threads write P into tensor memory and O += P V reads it from
// there as its A operand: only V comes from shared memory, which halves the
// shared-memory reads of that MMA.
//
// Roles (320 threads):
//   warp 0   producer: block-table entries -> TMA page loads into a ring of
//            64-key stages; a stage's K pages are stored [64-column block]
//            [page][16 rows][128 B] (V likewise), so that each 64-column
//            block of the tile is one uniformly strided swizzled operand;
//   warp 1   owns the tensor memory; one lane issues the MMAs;
//   warps 2-5 and 6-9  two softmax warpgroups, one thread per row
//            (tensor-memory lane).  Warpgroup w takes the tiles j with
//            j % 2 = w, with its own score buffer S[w], accumulator O[w] and
//            running (max, sum) per row (P buffers rotate), so the two
//            overlap; at the end warpgroup 0 merges the two (max, sum, O)
//            states of its row exactly (log-sum-exp) and stores the row.
// A warpgroup's reference max only moves when the row max grew by more
// than 2^8 (then its O row is rescaled in tensor memory): p <= 2^8, exact.
// Signals: S_j -> sbar[j % 2]; S_j read into registers -> sfree[j % 2] (128
// arrivals; S_{j+2} may then overwrite the buffer while the warpgroup is
// still working on tile j); P_j written -> pready[j % 2] (128 arrivals);
// O[j % 2] += P_j V_j done -> obar[j % 2]; the MMAs of tile j also release
// its stage (empty) and P buffer j % PBUFS (pfree).  A warp
// arrives on pready for its warpgroup's next tile only once that
// warpgroup's previous O += P V has completed (at most one phase ahead of
// the MMA lane).  The MMA lane polls both streams and issues whichever
// MMA is ready first.  Every wait is bounded; a timeout sets
// PKV_DEVERR_TIMEOUT and the CTA ends its work (the MMA lane waits for its
// own MMAs before tensor memory is freed).
constexpr int kURows = 128;                 // rows of an item: the MMA's M
constexpr int kUTileKeys = 64;              // keys of one stage
constexpr int kUTilePages = kUTileKeys / kPageRows;
constexpr int kUThreads = 10 * 32;
constexpr float kURescaleLog2 = 8.f;

// 16 columns of the warp's 32 tensor-memory lanes (one 32-bit value per
// lane and column).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

// D[tmem] (+)= A[tmem] . B[smem]: A read from tensor memory (see COL_P).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}
// N consecutive 32-bit columns of the warp's 32 lanes (N = 8 or 16).
template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&v)[N]) {
    static_assert(N == 8 || N == 16, "x8 or x16");
    if constexpr (N == 8) {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                         taddr),
                     "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                     "r"(v[7])
                     : "memory");
    } else {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
            "%13,%14,%15,%16};" ::"r"(taddr),
            "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
            "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
            "r"(v[15])
            : "memory");
    }
}

// N consecutive columns (N = 16 or 32), loaded or stored.
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&v)[N]) {
    if constexpr (N == 16) tmem_ld16(taddr, v);
    else tmem_ld32(taddr, v);
}
template <int N>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const uint32_t (&v)[N]) {
    if constexpr (N == 16) tmem_st<16>(taddr, v);
    else tmem_st32(taddr, v);
}

// Rows of an item split over T tensor-memory lanes each: an item of at most
// 128 / T query rows stores each row T times in the 128-row tile, in lane
// quadrants 4 / T apart, and the copy in quadrant group `part` takes the
// key columns [part 64 / T, (part + 1) 64 / T) of every tile with a softmax
// state of its own; the parts are merged at the end.  Half-full tiles then
// run their softmax on all four SM sub-partitions with half the columns per
// thread.
__host__ __device__ constexpr int umma_split(int rows) { return rows <= 32 ? 4 : (rows <= 64 ? 2 : 1); }

// NARROW (d = 64 only): a layout that lets two CTAs share an SM.  P is
// written over the scores it came from (tensor memory: 2 score/P buffers and
// 2 O accumulators, 256 columns) and the ring has 5 stages, so that two CTAs'
// shared memory and tensor memory fit one SM.
template <int D, bool NARROW = false>
struct ULayout {
    static_assert(!NARROW || D == 64, "the narrow layout is for d = 64");
    static constexpr int BOX = kPageRows * 128;                 // 16 rows x 64 bf16 columns
    static constexpr int NB = D / 64;                           // 64-column blocks of a row
    static constexpr int BLOCK_STRIDE = kUTilePages * BOX;      // between column blocks of a tile
    static constexpr int KV_BYTES = NB * BLOCK_STRIDE;          // one tile of K (or of V)
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;            // K tile, then V tile
    static constexpr int STAGES = NARROW ? 5 : (D == 64 ? 8 : 5);  // 80 / 128 / 160 KiB of ring
    static constexpr int Q_BLOCK = kURows * 128;                // one column block of Q
    static constexpr int OFF_Q = STAGES * STAGE_BYTES;
    static constexpr int PBUFS = 2;                             // P buffers, tile j uses j % 2
    static constexpr int OFF_XCHG = OFF_Q + NB * Q_BLOCK;       // (max, sum) of warpgroup 1's rows
    static constexpr int OFF_BAR = OFF_XCHG + kURows * 8;
    // full[STAGES], empty[STAGES], sbar[2], sfree[2], pready[2], obar[2], pfree[PBUFS],
    // mma_done, xchg, join, parts (split rows: the row's parts are staged)
    static constexpr int NBARS = 2 * STAGES + 12 + PBUFS;
    static constexpr int OFF_MASK = OFF_BAR + NBARS * 8;
    static constexpr int OFF_MISC = OFF_MASK + STAGES * 4;      // abort flag, TMEM base
    static constexpr size_t SMEM = 1024 + OFF_MISC + 16;
    static constexpr uint32_t COL_S = 0;                        // + 64 * warpgroup
    static constexpr uint32_t COL_O = 128;                      // + D * warpgroup
    // P buffer b: bf16 pairs of the hi part in columns [0, 32), of the lo
    // part in [32, 64) (lane = row, column c = keys 2c and 2c + 1: the A
    // operand layout of an MMA that reads A from tensor memory).  NARROW:
    // buffer b is score buffer b (tile j's P replaces its scores)
    static constexpr uint32_t COL_P = NARROW ? COL_S : COL_O + 2 * D;  // + 64 * buffer
    static constexpr uint32_t TMEM_COLS = NARROW ? 256 : 512;
    static_assert(COL_O + 2 * D <= TMEM_COLS && COL_P + 64 * PBUFS <= TMEM_COLS, "tensor memory");
    static constexpr uint32_t IDESC_S = umma_idesc_bf16(kURows, kUTileKeys, false);
    static constexpr uint32_t IDESC_O = umma_idesc_bf16(kURows, D, true);
};

struct UItem {
    int b;        // sequence whose block-table row lists the pages
    int h;        // kv head
    int t0, t1;   // the item's keys [t0, t1); t0 is page-aligned
    int npages;   // pages from t0 on that cover [t0, t1)
    int lo;       // no row reads a key before this one (V rows before it are zeroed)
};

struct URow {     // a softmax thread's row
    bool ok;
    const bf16* q;   // its query vector (D elements)
    int len, lo;     // it attends keys lo <= t < len
    void* out;       // the output row (D elements of out_bf16 ? bf16 : f32), or
    float* po;       // with out == nullptr: a partial, o (D floats) and
    float* pml;      // (max in log2 units, sum)
};

struct UArgs {
    const int32_t* block_tables;
    int32_t* err;
    int MB, Hkv, num_blocks, out_bf16;
    float scale_log2;
};

// Producer: the item's pages in 64-key stages (pages whose block id is out
// of range are skipped and reported).
template <int D, bool NARROW>
__device__ void umma_producer(const UArgs& a, const UItem& it, const CUtensorMap* tmk,
                              const CUtensorMap* tmv, uint8_t* base, uint64_t* full,
                              uint64_t* empty, uint32_t* masks, volatile int* s_abort) {
    using L = ULayout<D, NARROW>;
    const int lane = threadIdx.x & 31;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_parity[L::STAGES];
    uint32_t issued_any = 0;
    bool abort = false;
    const int32_t* row_tab = a.block_tables + (size_t)it.b * a.MB + it.t0 / kPageRows;
    int raw = lane < it.npages ? row_tab[lane] : -1;
    for (int c0 = 0; c0 < it.npages && !abort; c0 += 32) {
        int ent = -1;
        if (c0 + lane < it.npages) {
            if (raw < 0 || raw >= a.num_blocks)
                report_error(a.err, PKV_DEVERR_BLOCK_ID);
            else
                ent = raw;
        }
        raw = c0 + 32 + lane < it.npages ? row_tab[c0 + 32 + lane] : -1;
        const int cend = min(it.npages, c0 + 32);
        for (int s0 = c0; s0 < cend; s0 += kUTilePages) {
            const int npg = min(kUTilePages, it.npages - s0);
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
                mbar_arrive_expect_tx(&full[stage], __popc(vmask) * 2u * L::NB * L::BOX);
            }
            __syncwarp();
            if (mine) {
                uint8_t* kdst = base + stage * L::STAGE_BYTES + k * L::BOX;
                uint8_t* vdst = kdst + L::KV_BYTES;
                const int row0 = (ent * a.Hkv + it.h) * kPageRows;
#pragma unroll
                for (int bx = 0; bx < L::NB; ++bx) {
                    tma_load_2d(kdst + bx * L::BLOCK_STRIDE, tmk, bx * 64, row0, &full[stage]);
                    tma_load_2d(vdst + bx * L::BLOCK_STRIDE, tmv, bx * 64, row0, &full[stage]);
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
            report_error(a.err, PKV_DEVERR_TIMEOUT);
            for (int s = 0; s < L::STAGES; ++s)
                if (issued_any & (1u << s)) (void)mbar_wait(&full[s], issued_parity[s]);
        }
        __syncwarp();
    }
}

// The MMA lane.  Returns after its last MMA has completed (or it gave up).
template <int D, bool NARROW>
__device__ void umma_issuer(int ntiles, uint8_t* base, uint32_t tmem, uint64_t* full,
                            uint64_t* empty, uint64_t* sbar, uint64_t* sfree, uint64_t* pready,
                            uint64_t* obar, uint64_t* pfree, uint64_t* mma_done,
                            volatile int* s_abort, int32_t* err) {
    using L = ULayout<D, NARROW>;
    // Descriptors are built once and advanced by constant offsets: the start
    // address field holds address / 16 in its low bits (shared-memory
    // addresses stay below 2^18 bytes, so the sum never carries out of it).
    // One thread issues every MMA, so keeping its instruction chain short
    // sets how fast the tiles go.
    const uint64_t q_desc = umma_desc_sw128(smem_addr(base + L::OFF_Q), 16, 1024);
    const uint64_t k_desc0 = umma_desc_sw128(smem_addr(base), 16, 1024);
    const uint64_t v_desc0 = umma_desc_sw128(smem_addr(base + L::KV_BYTES), L::BLOCK_STRIDE, 1024);
    auto issue_s = [&](int j) {
        const int stage = j % L::STAGES;
        const uint64_t k_desc = k_desc0 + (uint64_t)((stage * L::STAGE_BYTES) >> 4);
        const uint32_t d = tmem + L::COL_S + 64u * (uint32_t)(j & 1);
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
            const uint64_t da = q_desc + (uint64_t)(((s >> 2) * L::Q_BLOCK + (s & 3) * 32) >> 4);
            const uint64_t db = k_desc + (uint64_t)(((s >> 2) * L::BLOCK_STRIDE + (s & 3) * 32) >> 4);
            umma_bf16(d, da, db, L::IDESC_S, s > 0);
        }
        umma_commit(&sbar[j & 1]);
    };
    auto issue_pv = [&](int j) {
        const int w = j & 1;
        const int stage = j % L::STAGES;
        const uint64_t v_desc = v_desc0 + (uint64_t)((stage * L::STAGE_BYTES) >> 4);
        const uint32_t pt = tmem + L::COL_P + (uint32_t)((j % L::PBUFS) * 64);
        const uint32_t o = tmem + L::COL_O + (uint32_t)(w * D);
#pragma unroll
        for (int s = 0; s < kUTileKeys / 16; ++s) {
            const uint64_t db = v_desc + (uint64_t)((s * 16 * 128) >> 4);
            umma_bf16_ts(o, pt + 8u * s, db, L::IDESC_O, j >= 2 || s > 0);
            umma_bf16_ts(o, pt + 32u + 8u * s, db, L::IDESC_O, true);
        }
        umma_commit(&obar[w]);
        umma_commit(&pfree[j % L::PBUFS]);
        umma_commit(&empty[stage]);  // the stage's K and V are no longer read
    };
    // S_j needs its stage loaded and (j >= 2) the buffer's previous scores read
    // (NARROW: O += P_{j-2} V_{j-2} issued, since that P sits where S_j goes;
    // the MMAs of this thread run in issue order, so P_{j-2} is read before
    // S_j overwrites it); PV_j needs P_j.  Neither condition can run two phases ahead of this lane
    // (the warpgroup's next arrivals wait for MMAs only this lane issues), so
    // each wait is on an unambiguous parity.  (Measured against this polling
    // loop: issuing every ready S first, and a fixed order S_{j+2}, PV_j after
    // each P_j with blocking waits, were both slower.)
    int js = 0, jp = 0;
    bool ok = true;
    uint64_t since = 0;
    uint32_t idle = 0;
    while (jp < ntiles) {
        bool progressed = false;
        const bool s_buf_free =
            js < 2 || (NARROW ? jp >= js - 1
                              : mbar_test_wait(&sfree[js & 1], (uint32_t)((js - 2) >> 1) & 1u));
        if (js < ntiles && s_buf_free &&
            mbar_test_wait(&full[js % L::STAGES], (uint32_t)(js / L::STAGES) & 1u)) {
            tc_fence_after();
            issue_s(js);
            ++js;
            progressed = true;
        }
        if (jp < js && mbar_test_wait(&pready[jp & 1], (uint32_t)(jp >> 1) & 1u)) {
            tc_fence_after();
            issue_pv(jp);
            ++jp;
            progressed = true;
        }
        if (progressed) {
            idle = 0;
            since = 0;
            continue;
        }
        // nothing ready: leave the issue slots of this sub-partition to the
        // softmax warps that share it for a moment before polling again
        __nanosleep(64);
        if ((++idle & 255u) == 0) {
            if (*s_abort) {
                ok = false;
                break;
            }
            const uint64_t now = global_timer_ns();
            if (since == 0) {
                since = now;
            } else if (now - since > kWaitLimitNs) {
                ok = false;
                break;
            }
        }
    }
    if (!ok) {
        *s_abort = 1;
        report_error(err, PKV_DEVERR_TIMEOUT);
    }
    // every MMA this lane issued has completed before tensor memory is freed
    umma_commit(mma_done);
    (void)mbar_wait(mma_done, 0);
}

// V rows of tile j that no row of the item may read (past the item's last
// key, or before the first key any row attends) may hold anything: a
// warpgroup's 128 threads zero them before P V reads them.
template <int D>
__device__ __forceinline__ void umma_zero_v_rows(const UItem& it, int j, int r, uint8_t* vt) {
    using L = ULayout<D>;
    const int tile_t0 = it.t0 + j * kUTileKeys;
    const int z_lo = max(0, it.lo - tile_t0), z_hi = min(kUTileKeys, it.t1 - tile_t0);
    if (z_lo <= 0 && z_hi >= kUTileKeys) return;
    for (int idx = r; idx < kUTileKeys * L::NB * 8; idx += kURows) {
        const int key = idx / (L::NB * 8), rest = idx % (L::NB * 8);
        if (key >= z_lo && key < z_hi) continue;
        const int nb = rest >> 3, ch = rest & 7;
        *reinterpret_cast<uint4*>(vt + nb * L::BLOCK_STRIDE + key * 128 + ch * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
}

// One item, run by all kUThreads threads of the CTA (every thread calls it;
// `row` matters to the softmax warps only).  T: tensor-memory lanes per
// query row (umma_split): the softmax thread of lane quadrant q takes the key
// columns of part q / (4 / T).
template <int D, int T, bool NARROW = false>
__device__ void umma_attend(const UArgs& a, const UItem& it, const URow& row,
                            const CUtensorMap* tmk, const CUtensorMap* tmv, uint8_t* base) {
    using L = ULayout<D, NARROW>;
    constexpr int NC = kUTileKeys / T;  // key columns of a tile per softmax thread
    // columns per tensor-memory access of O (narrow: half, for registers)
    constexpr int EC = NARROW ? 16 : 32;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L::OFF_BAR);
    uint64_t* empty = full + L::STAGES;
    uint64_t* sbar = empty + L::STAGES;
    uint64_t* sfree = sbar + 2;
    uint64_t* pready = sfree + 2;
    uint64_t* obar = pready + 2;
    uint64_t* pfree = obar + 2;
    uint64_t* mma_done = pfree + L::PBUFS;
    uint64_t* xchg_bar = mma_done + 1;
    uint64_t* join = xchg_bar + 1;
    uint64_t* parts_bar = join + 1;
    uint32_t* masks = reinterpret_cast<uint32_t*>(base + L::OFF_MASK);
    volatile int* s_abort = reinterpret_cast<volatile int*>(base + L::OFF_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L::OFF_MISC + 4);
    float2* xchg = reinterpret_cast<float2*>(base + L::OFF_XCHG);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = (it.npages + kUTilePages - 1) / kUTilePages;
    if (tid == 0) {
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sbar[i], 1);
            mbar_init(&sfree[i], kURows);
            mbar_init(&pready[i], kURows);
            mbar_init(&obar[i], 1);
        }
        for (int i = 0; i < L::PBUFS; ++i) mbar_init(&pfree[i], 1);
        mbar_init(mma_done, 1);
        mbar_init(xchg_bar, kURows);
        mbar_init(join, 2 * kURows);
        mbar_init(parts_bar, kURows);
        *s_abort = 0;
        fence_barrier_init();
    }
    const int r = 32 * (warp & 3) + lane;  // softmax threads: the row (tensor-memory lane)
    const int wg = (warp - 2) >> 2;        // softmax threads: the warpgroup
    const int part = (warp & 3) / (4 / T);  // softmax threads: the row's part
    if (warp >= 2) {
        // warpgroup 0 puts the Q rows into the swizzled tile (zeros for rows
        // past the item); the V halves of the ring start zeroed, so that a
        // key no row may read never holds a non-finite value when P = 0
        // multiplies it
        if (wg == 0) {
            const uint4* src = reinterpret_cast<const uint4*>(row.q);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 v = row.ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t off = (c >> 3) * L::Q_BLOCK + r * 128 + (((c & 7) ^ (r & 7)) << 4);
                *reinterpret_cast<uint4*>(base + L::OFF_Q + off) = v;
            }
        }
        for (int idx = tid - 64; idx < L::STAGES * L::KV_BYTES / 16; idx += 2 * kURows) {
            const int st = idx / (L::KV_BYTES / 16), w = idx % (L::KV_BYTES / 16);
            *reinterpret_cast<uint4*>(base + st * L::STAGE_BYTES + L::KV_BYTES + w * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    if (warp == 1) tmem_alloc(tmem_slot, L::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if constexpr (T > 1) {
        // split rows: a thread writes only its part's columns of its P rows;
        // the other columns stay zero for the whole item (warpgroup 0 clears
        // the P buffers of its lanes before any MMA can read them)
        if (warp >= 2 && warp < 6) {
            uint32_t z[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) z[e] = 0u;
            const uint32_t lb = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + L::COL_P;
#pragma unroll
            for (int c = 0; c < 64 * L::PBUFS; c += 16) tmem_st<16>(lb + (uint32_t)c, z);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (warp == 0) {
        umma_producer<D, NARROW>(a, it, tmk, tmv, base, full, empty, masks, s_abort);
        return;
    }
    if (warp == 1) {
        if (lane == 0) {
            umma_issuer<D, NARROW>(ntiles, base, tmem, full, empty, sbar, sfree, pready, obar, pfree,
                           mma_done, s_abort, a.err);
            (void)mbar_wait(join, 0);  // both warpgroups have read their O
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
        return;
    }

    // ---- softmax warpgroup wg: tiles j = wg, wg + 2, ... ----
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const uint32_t col_s = L::COL_S + 64u * (uint32_t)wg, col_o = L::COL_O + (uint32_t)(wg * D);
    const int row_len = row.ok ? row.len : 0;
    const int c_first = part * NC;  // this thread's first key column of a tile
    // a warp whose 32 rows are all padding (past the item's rows) has no
    // scores to read and no P worth writing: its rows of O are never stored.
    // It still keeps the tiles' cadence (the same waits and arrivals), so
    // that it never arrives for a later tile while an earlier one is open.
    const bool pad_warp = __all_sync(0xffffffffu, !row.ok);
    float m_used = kNegInfP, l_run = 0.f;
    bool ok = true;
    int k = 0;  // tiles this warpgroup has done
    for (int j = wg; j < ntiles; j += 2, ++k) {
        const int stage = j % L::STAGES;
        const bool w_ok = mbar_wait(&sbar[wg], (uint32_t)k & 1u) &&
                          mbar_wait(&full[stage], (uint32_t)(j / L::STAGES) & 1u) && !*s_abort;
        ok = __all_sync(0xffffffffu, w_ok);
        if (!ok) break;
        if (pad_warp) {
            tc_fence_before();
            mbar_arrive(&sfree[wg]);
            // one phase ahead of the MMAs at most (see below)
            if (k >= 1) {
                ok = __all_sync(0xffffffffu, mbar_wait(&obar[wg], (uint32_t)(k - 1) & 1u));
                if (!ok) break;
            }
            umma_zero_v_rows<D>(it, j, r, base + stage * L::STAGE_BYTES + L::KV_BYTES);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&pready[wg]);
            continue;
        }
        tc_fence_after();
        const uint32_t msk = masks[stage] >> (c_first / kPageRows);
        float x[NC];
        if constexpr (NC == 64) {
            uint32_t v0[32], v1[32];
            tmem_ld32(lane_base + col_s, v0);
            tmem_ld32(lane_base + col_s + 32, v1);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                x[e] = __uint_as_float(v0[e]);
                x[32 + e] = __uint_as_float(v1[e]);
            }
        } else if constexpr (NC == 32) {
            uint32_t v0[32];
            tmem_ld32(lane_base + col_s + (uint32_t)c_first, v0);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(v0[e]);
        } else {
            uint32_t v0[16];
            tmem_ld16(lane_base + col_s + (uint32_t)c_first, v0);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(v0[e]);
        }
        // the score buffer may take S_{j+2} now
        tc_fence_before();
        mbar_arrive(&sfree[wg]);
        const int tile_t0 = it.t0 + j * kUTileKeys + c_first;
        const int k_lo = max(0, row.lo - tile_t0), k_hi = min(NC, row_len - tile_t0);
        // the row maximum as a tree of eight independent chains
        float mx8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = kNegInfP;
        constexpr uint32_t kAllPages = (1u << (NC / kPageRows)) - 1u;
        if (k_lo == 0 && k_hi == NC && (msk & kAllPages) == kAllPages) {
#pragma unroll
            for (int e = 0; e < NC; ++e) {
                x[e] *= a.scale_log2;
                mx8[e & 7] = fmaxf(mx8[e & 7], x[e]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < NC; ++e) {
                const bool valid = e >= k_lo && e < k_hi && ((msk >> (e / kPageRows)) & 1u);
                x[e] = valid ? x[e] * a.scale_log2 : kNegInfP;
                mx8[e & 7] = fmaxf(mx8[e & 7], x[e]);
            }
        }
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float m_new = fmaxf(m_used, mx);
        const bool need = m_used != kNegInfP && m_new > m_used + kURescaleLog2;
        if (m_used == kNegInfP) m_used = m_new;
        if (__any_sync(0xffffffffu, need)) {
            // O += P_{j-2} V_{j-2}, this warpgroup's previous tile, has to
            // land before its O row is rescaled
            ok = __all_sync(0xffffffffu, mbar_wait(&obar[wg], (uint32_t)(k - 1) & 1u));
            if (!ok) break;
            tc_fence_after();
            const float alpha = need ? fast_exp2(m_used - m_new) : 1.f;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += EC) {
                uint32_t v[EC];
                tmem_ldn<EC>(lane_base + col_o + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < EC; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                tmem_stn<EC>(lane_base + col_o + c0, v);
            }
            tmem_wait_st();
            if (need) {
                l_run *= alpha;
                m_used = m_new;
            }
        }
        const float m_ref = m_used == kNegInfP ? 0.f : m_used;
        // P buffer j % PBUFS was last read by O += P_{j-PBUFS} V_{j-PBUFS}
        if (j >= L::PBUFS) {
            ok = __all_sync(0xffffffffu, mbar_wait(&pfree[j % L::PBUFS],
                                                   (uint32_t)(j / L::PBUFS - 1) & 1u));
            if (!ok) break;
            tc_fence_after();
        }
        // this thread's columns of P buffer j % PBUFS: hi pairs, then lo pairs
        const uint32_t p_col = lane_base + L::COL_P + (uint32_t)((j % L::PBUFS) * 64 + c_first / 2);
        float ps8[8];  // the row sum, eight independent chains
#pragma unroll
        for (int u = 0; u < 8; ++u) ps8[u] = 0.f;
        constexpr int CWMAX = NARROW ? 8 : 16;
        constexpr int CW = NC / 2 < CWMAX ? NC / 2 : CWMAX;  // words per tensor-memory store
#pragma unroll
        for (int c = 0; c < NC / 2; c += CW) {
            uint32_t hw[CW], lw[CW];
#pragma unroll
            for (int e = 0; e < CW; ++e) {
                const float p0 = fast_exp2(x[2 * (c + e)] - m_ref);
                const float p1 = fast_exp2(x[2 * (c + e) + 1] - m_ref);
                ps8[(2 * e) & 7] += p0;
                ps8[(2 * e + 1) & 7] += p1;
                hw[e] = pack_bf16(p0, p1);
                lw[e] = pack_bf16(p0 - bf16lo(hw[e]), p1 - bf16hi(hw[e]));
            }
            tmem_st<CW>(p_col + (uint32_t)c, hw);
            tmem_st<CW>(p_col + 32u + (uint32_t)c, lw);
        }
        if constexpr (NARROW && T > 1) {
            // P replaced the scores: the other parts' columns of this lane
            // still hold scores and must read as zero
            uint32_t z[CW];
#pragma unroll
            for (int e = 0; e < CW; ++e) z[e] = 0u;
            const uint32_t p_buf = lane_base + L::COL_P + (uint32_t)((j % L::PBUFS) * 64);
#pragma unroll
            for (int c = 0; c < 32; c += CW) {
                // warp-uniform: a warp is one part
                if (c >= c_first / 2 && c < c_first / 2 + NC / 2) continue;
                tmem_st<CW>(p_buf + (uint32_t)c, z);
                tmem_st<CW>(p_buf + 32u + (uint32_t)c, z);
            }
        }
        tmem_wait_st();
        l_run += ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
        umma_zero_v_rows<D>(it, j, r, base + stage * L::STAGE_BYTES + L::KV_BYTES);
        fence_proxy_async_smem();
        // O += P V of this warpgroup's previous tile has completed before
        // this warp arrives for the next: the warpgroup then runs at most one
        // phase ahead of the MMA lane, which keeps every parity wait on
        // pready, obar and pfree unambiguous (two phases ahead, a wait on
        // obar could mistake an older completed phase for the one it wants,
        // and a rescale could run under P V updates still in flight).  By now
        // that MMA has normally long finished.
        if (k >= 1) {
            ok = __all_sync(0xffffffffu, mbar_wait(&obar[wg], (uint32_t)(k - 1) & 1u));
            if (!ok) break;
        }
        tc_fence_before();
        mbar_arrive(&pready[wg]);
    }
    if (!ok) {
        *s_abort = 1;
        if (lane == 0) report_error(a.err, PKV_DEVERR_TIMEOUT);
    }
    // this warpgroup's tiles and its last O += P V
    const int n_mine = ntiles > wg ? (ntiles - wg + 1) / 2 : 0;
    const bool have_o =
        ok && n_mine > 0 &&
        __all_sync(0xffffffffu, mbar_wait(&obar[wg], (uint32_t)(n_mine - 1) & 1u));
    if (wg == 1) {
        xchg[r] = make_float2(have_o ? m_used : kNegInfP, have_o ? l_run : 0.f);
        mbar_arrive(xchg_bar);
        tc_fence_before();
        mbar_arrive(join);
        return;
    }
    // warpgroup 0: merge the two states of the lane, then (split rows) the
    // row's parts, then store the row
    const bool x_ok = __all_sync(0xffffffffu, mbar_wait(xchg_bar, 0));
    const float2 o1 = x_ok ? xchg[r] : make_float2(kNegInfP, 0.f);
    const int n1 = ntiles > 1 ? ntiles / 2 : 0;
    const bool have_o1 = x_ok && n1 > 0 && o1.x != kNegInfP;
    const float m0 = have_o ? m_used : kNegInfP;
    const float M = fmaxf(m0, have_o1 ? o1.x : kNegInfP);
    const float e0 = (have_o && m0 != kNegInfP) ? fast_exp2(m0 - M) : 0.f;
    const float e1 = have_o1 ? fast_exp2(o1.x - M) : 0.f;
    const float l_tot = (have_o ? l_run : 0.f) * e0 + (have_o1 ? o1.y : 0.f) * e1;
    const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
    const float w0 = e0 * inv, w1 = e1 * inv;
    if (__any_sync(0xffffffffu, have_o || have_o1)) tc_fence_after();
    const bool any_o = !pad_warp && __any_sync(0xffffffffu, have_o);
    const bool any_o1 = !pad_warp && __any_sync(0xffffffffu, have_o1);
    // split rows: part p > 0 leaves (max, sum) in xchg and its normalised
    // output in the ring's shared memory (every tile consumed); part 0 waits
    // for them and merges the parts exactly (log-sum-exp)
    // the ring's shared memory is free by now (every tile consumed)
    float* xo = reinterpret_cast<float*>(base);  // [lane][D]
    float M_all = M, l_all = l_tot;
    float sp[T];  // part 0: the weight of each part's normalised output
    sp[0] = 1.f;
    if constexpr (T > 1) {
        const bool parts_ok_in = ok && x_ok;
        if (part > 0) xchg[r] = make_float2(l_tot > 0.f ? M : kNegInfP, l_tot);
        if (part > 0 && !pad_warp) {  // warp-uniform: the tensor-memory loads are collective
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += EC) {
                uint32_t u0[EC], u1[EC];
                if (any_o) tmem_ldn<EC>(lane_base + L::COL_O + c0, u0);
                if (any_o1) tmem_ldn<EC>(lane_base + L::COL_O + D + c0, u1);
                if (any_o || any_o1) tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < EC; e += 4) {
                    float4 v;
                    float* vv = reinterpret_cast<float*>(&v);
#pragma unroll
                    for (int f = 0; f < 4; ++f) {
                        float t = any_o && w0 > 0.f ? __uint_as_float(u0[e + f]) * w0 : 0.f;
                        if (any_o1 && w1 > 0.f) t = fmaf(__uint_as_float(u1[e + f]), w1, t);
                        vv[f] = t;
                    }
                    *reinterpret_cast<float4*>(xo + (size_t)r * D + c0 + e) = v;
                }
            }
        }
        mbar_arrive(parts_bar);
        const bool p_ok = __all_sync(0xffffffffu, mbar_wait(parts_bar, 0)) && parts_ok_in;
        if (part == 0) {
            float mp[T], lp[T];
            mp[0] = l_tot > 0.f ? M : kNegInfP;
            lp[0] = l_tot;
#pragma unroll
            for (int q = 1; q < T; ++q) {
                const float2 st = p_ok ? xchg[r + 32 * q * (4 / T)] : make_float2(kNegInfP, 0.f);
                mp[q] = st.x;
                lp[q] = st.y;
            }
            M_all = kNegInfP;
#pragma unroll
            for (int q = 0; q < T; ++q) M_all = fmaxf(M_all, mp[q]);
            l_all = 0.f;
#pragma unroll
            for (int q = 0; q < T; ++q) {
                sp[q] = (lp[q] > 0.f && mp[q] != kNegInfP) ? lp[q] * fast_exp2(mp[q] - M_all) : 0.f;
                l_all += sp[q];
            }
            const float inv_all = l_all > 0.f ? 1.f / l_all : 0.f;
#pragma unroll
            for (int q = 0; q < T; ++q) sp[q] *= inv_all;
        }
    }
    const bool store = row.ok && part == 0;
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += EC) {
        float v[EC];
#pragma unroll
        for (int e = 0; e < EC; ++e) v[e] = 0.f;
        if (part == 0 && any_o) {
            uint32_t u[EC];
            tmem_ldn<EC>(lane_base + L::COL_O + c0, u);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < EC; ++e) v[e] = w0 > 0.f ? __uint_as_float(u[e]) * w0 : 0.f;
        }
        if (part == 0 && any_o1) {
            uint32_t u[EC];
            tmem_ldn<EC>(lane_base + L::COL_O + D + c0, u);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < EC; ++e)
                if (w1 > 0.f) v[e] = fmaf(__uint_as_float(u[e]), w1, v[e]);
        }
        if (!store) continue;
        if constexpr (T > 1) {
            // the parts' normalised outputs, weighted by their share of the row's sum
#pragma unroll
            for (int e = 0; e < EC; ++e) v[e] *= sp[0];
#pragma unroll
            for (int q = 1; q < T; ++q) {
                if (sp[q] == 0.f) continue;
                const float* src = xo + (size_t)(r + 32 * q * (4 / T)) * D + c0;
#pragma unroll
                for (int e = 0; e < EC; e += 4) {
                    const float4 t = *reinterpret_cast<const float4*>(src + e);
                    v[e] = fmaf(t.x, sp[q], v[e]);
                    v[e + 1] = fmaf(t.y, sp[q], v[e + 1]);
                    v[e + 2] = fmaf(t.z, sp[q], v[e + 2]);
                    v[e + 3] = fmaf(t.w, sp[q], v[e + 3]);
                }
            }
        }
        if (row.out && a.out_bf16) {
            uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(row.out) + c0);
#pragma unroll
            for (int e = 0; e < EC; e += 8)
                o[e / 8] = make_uint4(pack_bf16(v[e], v[e + 1]), pack_bf16(v[e + 2], v[e + 3]),
                                      pack_bf16(v[e + 4], v[e + 5]), pack_bf16(v[e + 6], v[e + 7]));
        } else {
            float4* o = reinterpret_cast<float4*>(row.out ? reinterpret_cast<float*>(row.out) + c0
                                                          : row.po + c0);
#pragma unroll
            for (int e = 0; e < EC; e += 4) o[e / 4] = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
    }
    if (store && !row.out) {
        row.pml[0] = l_all > 0.f ? M_all : kNegInfP;
        row.pml[1] = l_all;
    }
    tc_fence_before();
    mbar_arrive(join);
}

// Chunked prefill: item (sequence, kv head, row group of 128 rows,
// partition); row fr of the group is (query fr / G, head fr % G); query i
// sits at position L - C + i and attends keys up to it.  T = umma_split(C G)
// tensor-memory lanes per row.  NARROW (d = 64 with split rows, more items
// than SMs): the narrow layout lets two CTAs share an SM (at most 102
// registers a thread).
template <int D, int G, int T, bool NARROW>
__global__ void __launch_bounds__(kUThreads, NARROW ? 2 : 1)
    paged_prefill_umma_kernel(const __grid_constant__ PrefillParams p,
                              const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tm_k);
        prefetch_tensor_map(&tm_v);
    }
    grid_dependency_wait();
    grid_launch_dependents();
    // Longest first: CTAs start in blockIdx order, so the items of the
    // longest contexts go first and the last wave holds the short ones.
    // Every CTA ranks the lengths (the ring's memory is free until the item
    // starts).
    int* s_order = reinterpret_cast<int*>(base);
    int* s_len = s_order + p.B;
    const bool lpt = p.B <= kUThreads;
    if (lpt) {
        const int t = threadIdx.x;
        if (t < p.B) s_len[t] = p.context_lens[t];
        __syncthreads();
        if (t < p.B) {
            const int Lt = s_len[t];
            int rank = 0;
#pragma unroll 8
            for (int b2 = 0; b2 < p.B; ++b2) {
                const int L2 = s_len[b2];
                rank += (L2 > Lt) || (L2 == Lt && b2 < t);
            }
            s_order[rank] = t;
        }
        __syncthreads();
    }
    const PItem pit = prefill_item(p, lpt ? s_order : nullptr);
    if (pit.part >= pit.np) return;  // no keys in this partition (uniform: the whole CTA leaves)
    UItem it;
    it.b = pit.b;
    it.h = pit.h;
    it.t0 = pit.t0;
    it.t1 = pit.t1;
    it.npages = pit.npages;
    it.lo = pit.lo;
    URow row = {};
    if (warp >= 2) {
        // lane quadrant q holds rows (q mod 4/T) 32 + lane: each row T times
        const int fr = pit.rg * kURows + ((warp & 3) % (4 / T)) * 32 + lane;
        row.ok = fr < p.C * G;
        const int qi = row.ok ? fr / G : 0, hq = pit.h * G + (row.ok ? fr % G : 0);
        const size_t grow = ((size_t)pit.b * p.C + qi) * p.Hq + hq;
        row.q = p.q + grow * D;
        row.len = row.ok ? pit.L - p.C + qi + 1 : 0;
        row.lo = (p.window > 0 && row.len > p.window) ? row.len - p.window : 0;
        if (pit.np == 1) {
            row.out = p.out_bf16 ? (void*)(reinterpret_cast<bf16*>(p.out) + grow * D)
                                 : (void*)(reinterpret_cast<float*>(p.out) + grow * D);
        } else {
            row.out = nullptr;
            row.po = p.part_o + (grow * p.NP + pit.part) * D;
            row.pml = p.part_ml + (grow * p.NP + pit.part) * 2;
        }
    }
    UArgs a;
    a.block_tables = p.block_tables;
    a.err = p.err;
    a.MB = p.MB;
    a.Hkv = p.Hkv;
    a.num_blocks = p.num_blocks;
    a.out_bf16 = p.out_bf16;
    a.scale_log2 = p.scale_log2;
    umma_attend<D, T, NARROW>(a, it, row, &tm_k, &tm_v, base);
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
    int window;        // sliding window (0: none)
    int split;         // tensor-memory lanes per row (umma_split of the largest group's rows)
    float scale_log2;
};

// Context length of sequence b, clamped as the decode clamps it.
__device__ __forceinline__ int cascade_len(const CascadeParams& p, int b) {
    const int L = p.context_lens[b];
    const int maxlen = p.MB * kPageRows;
    return L < 0 ? 0 : (L > maxlen ? maxlen : L);
}

// Shared tokens of sequence b as the decode counts them: whole pages inside
// its (clamped) context.
__device__ __forceinline__ int cascade_shared(const CascadeParams& p, int b) {
    const int L = cascade_len(p, b);
    const int s = p.shared_tokens[b];
    return s < 0 ? 0 : (s > L ? L : s) / kPageRows * kPageRows;
}

// First token sequence b's query attends (sliding window; 0 otherwise).
__device__ __forceinline__ int cascade_lo(const CascadeParams& p, int b) {
    const int L = cascade_len(p, b);
    return (p.window > 0 && L > p.window) ? L - p.window : 0;
}

// One CTA per (group, kv head, row group of 128 rows): the rows are
// (member, head) pairs, member m of the group and head g -> row m*G + g;
// every row attends to the first shared_tokens of its own sequence (under a
// sliding window only those inside its window: a row whose window starts past
// them leaves an empty partial), read
// once for the group from the pages of the member that shares the most (the
// others' shared block-table entries must be the same ids: a mismatch sets
// PKV_DEVERR_PREFIX).  The tiles run on the tensor cores (umma_attend).  The
// result goes to partial slot 0 of each member; the decode kernel writes the
// rest of the sequence to slots 1.. and the combine merges them.  The kernel
// does not wait for the decode kernel before it starts (it reads nothing the
// decode writes; q was rotated before the decode began), so its CTAs fill
// SMs as the decode's CTAs finish; each CTA waits for the decode grid before
// it exits, so that the combine, which waits for this grid, also sees the
// decode's partials.  T = p.split; NARROW as for the prefill (two CTAs per
// SM at d = 64 with split rows).
template <int D, int G, int T, bool NARROW>
__global__ void __launch_bounds__(kUThreads, NARROW ? 2 : 1)
    cascade_prefix_kernel(const __grid_constant__ CascadeParams p,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    // first member, member count, leader, the leader's shared tokens, the
    // first token any row attends
    __shared__ int s_grp[5];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_launch_dependents();
    int x = blockIdx.x;
    const int rg = x % p.RG;
    x /= p.RG;
    const int h = x % p.Hkv, g = x / p.Hkv;
    if (tid == 0) {
        int gs = p.group_start[g], ge = p.group_start[g + 1];
        if (gs < 0 || ge < gs || ge > p.B) {
            report_error(p.err, PKV_DEVERR_PREFIX);
            gs = ge = 0;
        }
        int best = 0, leader = gs, minlo = INT_MAX;
        for (int b = gs; b < ge; ++b) {
            const int sb = cascade_shared(p, b), lo = cascade_lo(p, b);
            if (sb > best) {
                best = sb;
                leader = b;
            }
            if (lo < sb) minlo = min(minlo, lo);
        }
        s_grp[0] = gs;
        s_grp[1] = ge - gs;
        s_grp[2] = leader;
        s_grp[3] = best;
        // no row has a shared token inside its window: one page, all masked
        s_grp[4] = minlo < best ? minlo : max(best - 1, 0);
    }
    __syncthreads();
    const int gs = s_grp[0], nmem = s_grp[1], leader = s_grp[2], S = s_grp[3];
    const int first_key = s_grp[4];
    if (S > 0 && rg * kURows < nmem * G) {
        if (warp == 0 && lane == 0) {
            prefetch_tensor_map(&tm_k);
            prefetch_tensor_map(&tm_v);
        }
        // every member's shared pages must be the leader's (checked once, by row group 0)
        if (rg == 0 && h == 0) {
            for (int idx = tid; idx < nmem * (S / kPageRows); idx += kUThreads) {
                const int m = idx / (S / kPageRows), j = idx - m * (S / kPageRows);
                const int b = gs + m;
                if (j < cascade_shared(p, b) / kPageRows &&
                    p.block_tables[(size_t)b * p.MB + j] != p.block_tables[(size_t)leader * p.MB + j])
                    report_error(p.err, PKV_DEVERR_PREFIX);
            }
        }
        UItem it;
        it.b = leader;
        it.h = h;
        // pages before the page of the first key any row attends are skipped
        it.t0 = first_key / kPageRows * kPageRows;
        it.t1 = S;
        it.npages = (S - it.t0) / kPageRows;
        it.lo = first_key;
        URow row = {};
        if (warp >= 2) {
            const int fr = rg * kURows + ((warp & 3) % (4 / p.split)) * 32 + lane;
            const int m = fr / G, hq = h * G + fr % G;
            const int b = gs + m;
            row.len = m < nmem ? cascade_shared(p, b) : 0;
            row.ok = row.len > 0;  // no shared tokens: no slot 0
            row.lo = m < nmem ? cascade_lo(p, b) : 0;
            const size_t r = (size_t)(row.ok ? b : 0) * p.Hq + hq;
            row.q = p.q + r * D;
            row.out = nullptr;
            row.po = p.part_o + (r * p.NPT) * D;
            row.pml = p.part_ml + (r * p.NPT) * 2;
        }
        UArgs a;
        a.block_tables = p.block_tables;
        a.err = p.err;
        a.MB = p.MB;
        a.Hkv = p.Hkv;
        a.num_blocks = p.num_blocks;
        a.out_bf16 = 0;
        a.scale_log2 = p.scale_log2;
        umma_attend<D, T, NARROW>(a, it, row, &tm_k, &tm_v, base);
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

// The tensor-core (tcgen05) prefill: one 128-row item per CTA; one CTA per
// SM, two with the narrow layout.
template <int D, int G, int T, bool NARROW>
cudaError_t launch_prefill_umma_split(const PrefillArgs& a, const CUtensorMap& tmk,
                                      const CUtensorMap& tmv) {
    using L = ULayout<D, NARROW>;
    auto kern = paged_prefill_umma_kernel<D, G, T, NARROW>;
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
    p.RG = (int)((a.C * G + kURows - 1) / kURows);
    p.num_blocks = (int)a.num_blocks;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out_bf16 = a.out_dtype == PKV_DTYPE_BF16;
    p.window = a.window;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.Hkv * p.RG * a.max_partitions));
    cfg.blockDim = dim3(kUThreads);
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

// Two CTAs per SM pay where the items outnumber the SMs (at batch 1, 64
// items on 148 SMs, a shared SM only slows its pair: 16.1 -> 16.9 us).
template <int D, int G>
cudaError_t launch_prefill_umma_typed(const PrefillArgs& a, const CUtensorMap& tmk,
                                      const CUtensorMap& tmv) {
    const int64_t items =
        a.B * a.Hkv * ((a.C * G + kURows - 1) / kURows) * (int64_t)a.max_partitions;
    const bool narrow = D == 64 && items > (int64_t)device_sm_count();
    switch (umma_split((int)(a.C * G))) {
        case 4:
            return narrow ? launch_prefill_umma_split<D, G, 4, (D == 64)>(a, tmk, tmv)
                          : launch_prefill_umma_split<D, G, 4, false>(a, tmk, tmv);
        case 2:
            return narrow ? launch_prefill_umma_split<D, G, 2, (D == 64)>(a, tmk, tmv)
                          : launch_prefill_umma_split<D, G, 2, false>(a, tmk, tmv);
        default: return launch_prefill_umma_split<D, G, 1, false>(a, tmk, tmv);
    }
}

template <int D>
cudaError_t prefill_dispatch_g(const PrefillArgs& a, const CUtensorMap& k, const CUtensorMap& v) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_prefill_umma_typed<D, 1>(a, k, v);
        case 2: return launch_prefill_umma_typed<D, 2>(a, k, v);
        case 4: return launch_prefill_umma_typed<D, 4>(a, k, v);
        case 8: return launch_prefill_umma_typed<D, 8>(a, k, v);
    }
    return cudaErrorInvalidValue;
}

template <int D, int G, int T, bool NARROW>
cudaError_t launch_cascade_split(const CascadeArgs& a, const CUtensorMap& tmk,
                                 const CUtensorMap& tmv) {
    using L = ULayout<D, NARROW>;
    auto kern = cascade_prefix_kernel<D, G, T, NARROW>;
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
    p.window = a.window;
    p.RG = (int)((a.max_group_size * G + kURows - 1) / kURows);
    p.split = umma_split((int)(a.max_group_size * G));
    p.NG = (int)a.num_groups;
    p.num_blocks = (int)a.num_blocks;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.num_groups * a.Hkv * p.RG));
    cfg.blockDim = dim3(kUThreads);
    cfg.dynamicSmemBytes = L::SMEM;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p, tmk, tmv);
}

template <int D, int G>
cudaError_t launch_cascade_typed(const CascadeArgs& a, const CUtensorMap& tmk,
                                 const CUtensorMap& tmv) {
    const int64_t items = a.num_groups * a.Hkv * ((a.max_group_size * G + kURows - 1) / kURows);
    const bool narrow = D == 64 && items > (int64_t)device_sm_count();
    switch (umma_split((int)(a.max_group_size * G))) {
        case 4:
            return narrow ? launch_cascade_split<D, G, 4, (D == 64)>(a, tmk, tmv)
                          : launch_cascade_split<D, G, 4, false>(a, tmk, tmv);
        case 2:
            return narrow ? launch_cascade_split<D, G, 2, (D == 64)>(a, tmk, tmv)
                          : launch_cascade_split<D, G, 2, false>(a, tmk, tmv);
        default: return launch_cascade_split<D, G, 1, false>(a, tmk, tmv);
    }
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
