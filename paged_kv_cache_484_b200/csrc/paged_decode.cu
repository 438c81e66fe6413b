// paged_decode.cu -- single-query attention over a paged KV cache on sm_100a.
//
// What it computes ("Inference From Scratch", ch. 8 online softmax and ch. 10
// paged attention / block tables; "The Project: Serve Your Own LLM", M2 GQA):
// for every sequence b and query head h, softmax(q K^T * scale) V over the
// context_lens[b] tokens that block_tables[b] lists, in fp32.
//
// Work decomposition.  A work item is (sequence, kv head, partition): the
// partition is P consecutive tokens of the sequence (P chosen on the host),
// and one item serves all G = Hq / Hkv query heads of the kv head, so every
// K/V page is read from HBM once per step.  The grid is persistent (a
// multiple of the SM count); every CTA first turns context_lens into an
// exclusive prefix of partition counts in shared memory, then walks items
// i = blockIdx.x, blockIdx.x + gridDim.x, ...  Sequences that need one
// partition write their output directly; longer ones write a partial
// (running max, sum, normalised output) that the combine kernel merges
// ("flash-decoding" split-K; the pages do not describe it, the log-sum-exp
// merge below is exact up to rounding).
//
// Inside a CTA.  One producer warp reads the block-table entries (one lane
// per page, prefetched a chunk ahead), and issues TMA tensor loads of each
// 16-token K page and V page into a ring of shared-memory stages, signalled
// by mbarriers with transaction counts; the q rows of the item ride along
// with the item's first stage as a bulk copy.  Four consumer warps each take
// one page per stage:
//   * bf16 (default): S = Q K^T and O += P V on the tensor cores with
//     mma.sync m16n8k16 (bf16 in, fp32 accumulate).  The G query heads are
//     rows of the 16-row A tile; rows G..2G-1 repeat them so that the same
//     MMA yields a second copy of the scores, which those rows turn into the
//     low part of a two-term bf16 split of P (p = hi + lo, |p - hi - lo| <=
//     2^-17 p), keeping P V accurate to fp32 level although the MMA takes
//     bf16 operands.  K/V are read with ldmatrix from 128-byte-swizzled
//     pages (bank-conflict free).
//   * fp32 inputs, or bf16 with PKV_DECODE_FORCE_SIMT: CUDA cores; lanes of a
//     token group each hold 16 bytes of the row, q.k partial sums are reduced
//     with warp shuffles, and each token group keeps its own online softmax.
// At the end of an item the consumer warps merge their (max, sum, output)
// triples through shared memory and write the result.
//
// Every wait is bounded (PKV_DEVERR_TIMEOUT); block ids and context lengths
// are range-checked (PKV_DEVERR_BLOCK_ID / _CONTEXT_LEN) and the bad page or
// length is skipped or clamped instead of being dereferenced.
#include <cuda_bf16.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

using bf16 = __nv_bfloat16;
constexpr int NW = kConsumerWarps;
constexpr float kNegInf = -__builtin_huge_valf();
// Batches of at most this many sequences hand out every sequence's last
// (shortest) partition after all full ones, longest first, so that the
// work that finishes last is short.
constexpr int kLptMaxSeqs = 256;
// cascade offsets live in the longest-first arrays' shared memory
static_assert(kCascadeMaxSeqs <= kLptMaxSeqs, "cascade offsets need the rank arrays");

__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }
__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Tag for the 8-bit cache: E4M3 codes times a per-tensor scale (q stays
// bf16).  Its K pages keep the [16 tokens][D] row layout; its V pages are
// stored transposed, [D][16 tokens], so that the four tokens one lane needs
// for the output MMA are four consecutive bytes.  A page's K codes and V
// codes are one contiguous region of the cache ([K | V] per (block, kv
// head)), which one TMA box fetches at d = 64.
struct e4m3kv {};

template <typename T, int D, int G>
struct Layout {
    static constexpr bool F8 = std::is_same<T, e4m3kv>::value;
    static constexpr int ESZ = F8 ? 1 : (int)sizeof(T);             // cache element bytes
    static constexpr int QSZ = F8 ? 2 : (int)sizeof(T);             // q element bytes
    static constexpr bool SWZ = std::is_same<T, bf16>::value;  // 128B-swizzled bf16 pages
    // 8-bit K pages with 128-byte rows are 128B-swizzled too (bank-conflict
    // free 16-byte row reads); 64-byte rows need no swizzle.
    static constexpr bool SWZ_K8 = F8 && D == 128;
    static constexpr int ROW_BYTES = D * ESZ;
    static constexpr int PAGE_BYTES = kPageRows * ROW_BYTES;
    static constexpr int BOXES = SWZ ? D / 64 : 1;  // TMA boxes per page
    static constexpr int BOX_BYTES = PAGE_BYTES / BOXES;
    // Pages each consumer warp takes per stage: two for the d = 64 tensor-core
    // paths with G <= 4 (a 32-token tile: longer independent MMA chains and
    // half the softmax bookkeeping per token; the 8-bit cache at G = 8 too),
    // else one.
    static constexpr int PPW = ((SWZ && D == 64 && G <= 4) || (F8 && D == 64)) ? 2 : 1;
    static constexpr int STAGE_PAGES = NW * PPW;
    static constexpr int STAGE_BYTES = 2 * STAGE_PAGES * PAGE_BYTES;
    // Where a stage's pages sit: page k's K at k * KPITCH, its V VOFF past
    // that.  The 8-bit cache keeps a page's K and V together ([K | V] per
    // page, as in the cache); the others place a stage's K pages, then its V
    // pages.
    static constexpr int KPITCH = F8 ? 2 * PAGE_BYTES : PAGE_BYTES;
    static constexpr int VOFF = F8 ? PAGE_BYTES : STAGE_PAGES * PAGE_BYTES;
    // 64 KiB of ring (96 KiB for bf16 d = 128, whose CTAs are two per SM
    // by registers anyway)
    static constexpr int STAGES =
        cmax(2, cmin(6, ((D == 128 && SWZ) ? 98304 : 65536) / STAGE_BYTES));
    static constexpr int Q_COPY = G * D * QSZ;
    static constexpr int Q_BYTES = round_up(Q_COPY, 128);
    static constexpr int ROW_COPY = D * QSZ;           // one new k or v row (q's type)
    // fused step: the raw new k row and v row, or (8-bit cache) their codes,
    // computed by the producer
    static constexpr int NEWKV_BYTES = F8 ? 2 * D : 2 * ROW_COPY;
    // Item merge: each warp leaves (o[D], m, l) per head in its own K and V
    // page slots of the item's last stage (free once it has read its pages),
    // or, where those are too small (8-bit d = 128 at G = 8), in a region of
    // its own.
    static constexpr int MERGE_ROW_BYTES = (D + 2) * 4;
    static constexpr int MERGE_ROWS_PER_SLOT = PPW * PAGE_BYTES / MERGE_ROW_BYTES;
    static constexpr bool MERGE_IN_SLOTS = 2 * MERGE_ROWS_PER_SLOT >= G;
    // With a region of its own the item's last stage goes back to the
    // producer before the merge, and the warps meet once more after it.
    static constexpr bool MERGE_SEPARATE = !MERGE_IN_SLOTS;
    static constexpr int MERGE_BYTES = MERGE_SEPARATE ? NW * G * MERGE_ROW_BYTES : 0;
    // byte offsets from the 1024-aligned base
    static constexpr int OFF_Q = STAGES * STAGE_BYTES;
    static constexpr int OFF_NEWKV = OFF_Q + STAGES * Q_BYTES;
    // fused step: per stage, cos[D/2], sin[D/2] (fp32) of the item's position,
    // written by the producer with the item's first stage
    static constexpr int ROPE_BYTES = D * 4;
    static constexpr int OFF_ROPE = OFF_NEWKV + STAGES * NEWKV_BYTES;
    static constexpr int OFF_MERGE = OFF_ROPE + STAGES * ROPE_BYTES;
    static constexpr int OFF_BAR = OFF_MERGE + MERGE_BYTES;
    // full, empty, q per stage; merge; rank (the longest-first order is ready)
    static constexpr int OFF_MASK = OFF_BAR + (3 * STAGES + 2) * 8;
    // Cluster mode: every CTA of a cluster stores its merged partial (o[D], m,
    // l per head) into slot `rank` of a landing area in rank 0's shared memory,
    // past everything else (rank 0 may still be computing when they land).
    static constexpr int CLUSTER_PART_BYTES = G * (D + 2) * 4;
    static constexpr int OFF_PATCH = OFF_MASK + STAGES * 4;  // fused: (row, block) of the new token
    static constexpr int OFF_ITEM = OFF_PATCH + STAGES * 8;  // work item of each stage, -1: no more
    // abort flag, per-warp counts of non-empty contexts, 8 scan slots
    static constexpr int OFF_MISC = OFF_ITEM + STAGES * 4;
    // s_len[B], s_pre[B + 1]; with at most kLptMaxSeqs sequences also
    // s_rank[B], s_key[B] (the longest-first order of last partitions)
    static constexpr int OFF_SEQ = OFF_MISC + 16 * 4;
    static size_t smem_bytes(int B) {
        return 1024 + OFF_SEQ + (size_t)(2 * B + 1) * 4 + (B <= kLptMaxSeqs ? (size_t)2 * B * 4 : 0);
    }
    // cluster mode: the landing area (16-byte aligned, after the sequence arrays)
    __host__ __device__ static constexpr int land_offset(int B) {
        return round_up(OFF_SEQ + (2 * B + 1) * 4 + (B <= kLptMaxSeqs ? 2 * B * 4 : 0), 16);
    }
    static size_t cluster_smem_bytes(int B, int cs) {
        return 1024 + (size_t)land_offset(B) + (size_t)cs * CLUSTER_PART_BYTES;
    }
};

struct DecodeParams {
    const void* q;
    const int32_t* block_tables;
    const int32_t* context_lens;
    void* out;
    float* part_o;
    float* part_ml;
    int32_t* err;
    // item counter and finished-CTA counter (zero before the launch, zero
    // after it); null: items are dealt out round-robin instead
    uint32_t* sched;
    int B, Hq, Hkv, MB, P, NP;
    int num_blocks;
    float scale_log2;  // softmax scale x log2(e) (x k_scale for the 8-bit cache)
    float v_scale;     // 8-bit cache: V = code x v_scale; 1 otherwise
    float k_scale;     // 8-bit cache: K = code x k_scale (the fused step's new codes)
    int out_bf16;
    // cluster mode: CS > 1 CTAs per (sequence, kv head), CTA rank r takes
    // partition r, and the cluster merges the partials in shared memory
    // (no workspace partials, no combine kernel); 0 = off
    int cluster;
    // cascade: the first shared_tokens[b] tokens of sequence b are attended by
    // the shared-prefix pass (partial slot 0); this kernel takes the rest,
    // in partitions that start at that offset (slots 1..); null = off
    const int32_t* shared_tokens;
    // sliding window: each query attends to the last `window` tokens of its
    // context (0 = the whole context)
    int window;
    // fused step only: the new token of every sequence (q's type)
    const void* k_new;            // [B, Hkv, D]
    const void* v_new;            // [B, Hkv, D]
    const int64_t* positions;     // [B]
    const int64_t* slot_mapping;  // [B]
    void* k_cache;                // cache bases for the new rows (8-bit: the [K | V] pages)
    void* v_cache;
};

struct RopeFreq {
    double f[64];  // theta^(-2i/d), i < d/2 (fused step)
};

struct Item {
    int b, h, part, t0, t1, npages, np;
    int slot0;  // cascade: 1 when the sequence's shared prefix owns partial slot 0
    int lo;     // first token attended (sliding window; 0 otherwise)
};

// Sliding window: first token a context of Lb tokens attends to, and the
// start of its page (where the sequence's partitions begin).
__host__ __device__ __forceinline__ int window_start(int window, int Lb) {
    return (window > 0 && Lb > window) ? Lb - window : 0;
}
__host__ __device__ __forceinline__ int window_page_start(int window, int Lb) {
    return window_start(window, Lb) / kPageRows * kPageRows;
}

// Item i -> (sequence, kv head, partition).  Items are j * Hkv + h.  Without
// the longest-first order, j runs over every sequence's partitions in order
// (s_pre: exclusive prefix of partition counts).  With it (p.B <=
// kLptMaxSeqs), j < s_pre[B] runs over the partitions before each sequence's
// last one, and j >= s_pre[B] over the last partitions in the order s_rank.
__device__ __forceinline__ Item decode_item(int i, const DecodeParams& p, const int* s_len,
                                            const int* s_pre) {
    Item it;
    const int j = i / p.Hkv;
    it.h = i - j * p.Hkv;
    const int nfull = s_pre[p.B];
    if (p.B <= kLptMaxSeqs && !p.cluster && !p.shared_tokens && j >= nfull) {
        const int* s_rank = s_pre + p.B + 1;
        it.b = s_rank[j - nfull];
        it.np = (s_len[it.b] - window_page_start(p.window, s_len[it.b]) + p.P - 1) / p.P;
        it.part = it.np - 1;
    } else {
        int lo = 0, hi = p.B - 1;  // largest b with s_pre[b] <= j
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_pre[mid] <= j) lo = mid;
            else hi = mid - 1;
        }
        it.b = lo;
        it.part = j - s_pre[lo];
        it.np = (s_len[lo] - window_page_start(p.window, s_len[lo]) + p.P - 1) / p.P;
    }
    // sliding window: partitions start at the page of the window's first token
    int off = window_page_start(p.window, s_len[it.b]);
    it.lo = window_start(p.window, s_len[it.b]);
    it.slot0 = 0;
    if (p.shared_tokens) {
        // cascade: partitions start after the tokens of the shared-prefix pass
        // (or at the window's page, when the window starts past them); slot 0
        // belongs to the shared prefix whenever it has tokens
        const int sh = (s_pre + p.B + 1)[it.b];
        off = max(sh, off);
        it.np = (s_len[it.b] - off + p.P - 1) / p.P;
        it.slot0 = sh > 0 ? 1 : 0;
    }
    it.t0 = off + it.part * p.P;
    it.t1 = min(s_len[it.b], it.t0 + p.P);
    it.npages = (it.t1 - it.t0 + kPageRows - 1) / kPageRows;
    return it;
}

// Byte offset of 16-byte chunk `c` of token row `tok` inside a staged page.
template <typename T, int D>
__device__ __forceinline__ uint32_t chunk_offset(int tok, int c) {
    if constexpr (std::is_same<T, bf16>::value) {
        // TMA SWIZZLE_128B: chunk index XOR (row % 8) inside each 128-byte row;
        // D = 128 pages are two 64-column boxes of 2 KiB each.
        if constexpr (D == 64) {
            return tok * 128 + ((c ^ (tok & 7)) << 4);
        } else {
            return (c >> 3) * 2048 + tok * 128 + (((c & 7) ^ (tok & 7)) << 4);
        }
    } else {
        return tok * (D * (int)sizeof(T)) + (c << 4);
    }
}

__device__ __forceinline__ void store_out(void* out, size_t idx, float v, int out_bf16) {
    if (out_bf16)
        reinterpret_cast<bf16*>(out)[idx] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float*>(out)[idx] = v;
}


// ---- fused step: RoPE on the new token inside the decode kernel ------------
// Same arithmetic as kv_append.cu: fp64 angle, sine/cosine and rotation, one
// rounding to the storage type.

template <typename T>
__device__ __forceinline__ double to_d(T x);
template <>
__device__ __forceinline__ double to_d<float>(float x) { return (double)x; }
template <>
__device__ __forceinline__ double to_d<bf16>(bf16 x) { return (double)__bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_d(double x);
template <>
__device__ __forceinline__ float from_d<float>(double x) { return __double2float_rn(x); }
template <>
__device__ __forceinline__ bf16 from_d<bf16>(double x) {
    const uint16_t b = double_to_bf16_bits(x);
    return *reinterpret_cast<const bf16*>(&b);
}

// Fused step: the cos/sin table of a position, tab[i] = cos(pos f_i),
// tab[D/2 + i] = sin(pos f_i), i < D/2: angle in fp64, reduced mod 2pi in
// fp64, then sine and cosine in fp32 of the reduced angle; `f` holds
// theta^(-2i/d) for the lane's i = lane + 32 u.  A warp computes its lanes'
// entries into registers (cs[u], sn[u]) ahead of time, and stores them when
// the stage that carries them is issued.
template <int D>
__device__ __forceinline__ void warp_rope_regs(double pos, const double (&f)[(D + 63) / 64],
                                               float (&cs)[(D + 63) / 64],
                                               float (&sn)[(D + 63) / 64]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int u = 0; u < (D + 63) / 64; ++u) {
        cs[u] = 1.f;
        sn[u] = 0.f;
        if (lane + 32 * u < D / 2) sincosf((float)reduce_two_pi(pos * f[u]), &sn[u], &cs[u]);
    }
}
template <int D>
__device__ __forceinline__ void warp_rope_store(const float (&cs)[(D + 63) / 64],
                                                const float (&sn)[(D + 63) / 64], float* tab) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int u = 0; u < (D + 63) / 64; ++u) {
        const int i = lane + 32 * u;
        if (i < D / 2) {
            tab[i] = cs[u];
            tab[D / 2 + i] = sn[u];
        }
    }
}

// Element `col` of the rotated row (row in storage type T); the pair partner
// is col +- D/2.  fp32 arithmetic (the result is rounded to T by the caller).
template <typename T, int D>
__device__ __forceinline__ float rotated_elem(const T* row, int col, const float* tab) {
    constexpr int HALF = D / 2;
    const int i = col < HALF ? col : col - HALF;
    const float x = (float)to_d<T>(row[col]);
    const float y = (float)to_d<T>(row[col < HALF ? col + HALF : col - HALF]);
    return col < HALF ? fmaf(x, tab[i], -y * tab[HALF + i]) : fmaf(x, tab[i], y * tab[HALF + i]);
}

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// One warp writes the new token's rotated k row and raw v row into row r of
// the staged K and V pages (overwriting what the TMA brought) and into the
// cache rows in global memory; then orders its shared-memory writes before
// any later TMA write into the same stage.
// Out of line: it runs once per sequence, and inlined into the consumers'
// page loop it cost the fused d = 64 kernel 6 registers and a spill (ragged
// batch 56.6 -> 55.5 us out of line).
template <typename T, int D>
__device__ __noinline__ void patch_new_row(uint8_t* kpage, uint8_t* vpage, const uint8_t* newkv, int r,
                              const float* tab, T* kglob, T* vglob) {
    constexpr int HALF = D / 2, E = 16 / (int)sizeof(T), CH = D * (int)sizeof(T) / 16;
    const int lane = threadIdx.x & 31;
    const T* kn = reinterpret_cast<const T*>(newkv);
    const uint8_t* vn = newkv + D * sizeof(T);
    for (int i = lane; i < HALF; i += 32) {
        const int i1 = i + HALF;
        const T y0 = from_f<T>(rotated_elem<T, D>(kn, i, tab));
        const T y1 = from_f<T>(rotated_elem<T, D>(kn, i1, tab));
        *reinterpret_cast<T*>(kpage + chunk_offset<T, D>(r, i / E) + (i % E) * sizeof(T)) = y0;
        *reinterpret_cast<T*>(kpage + chunk_offset<T, D>(r, i1 / E) + (i1 % E) * sizeof(T)) = y1;
        kglob[i] = y0;
        kglob[i1] = y1;
    }
    for (int c = lane; c < CH; c += 32) {
        const uint4 v = *reinterpret_cast<const uint4*>(vn + c * 16);
        *reinterpret_cast<uint4*>(vpage + chunk_offset<T, D>(r, c)) = v;
        reinterpret_cast<uint4*>(vglob)[c] = v;
    }
    __syncwarp();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The same for the 8-bit cache, whose codes the producer has computed
// (k codes at newkv[0, D), v codes at newkv[D, 2D)) and already written to
// the cache: copy them into row r of the staged K half (128-byte rows are
// 128B-swizzled at d = 128) and column r of the transposed V half.
template <int D>
__device__ __forceinline__ void patch_new_codes(uint8_t* kpage, uint8_t* vpage,
                                                const uint8_t* newkv, int r) {
    const int lane = threadIdx.x & 31;
    if (lane < D / 16) {
        const int c = D == 128 ? (lane ^ (r & 7)) : lane;
        *reinterpret_cast<uint4*>(kpage + r * D + c * 16) =
            *reinterpret_cast<const uint4*>(newkv + lane * 16);
    }
    for (int i = lane; i < D; i += 32) vpage[i * kPageRows + r] = newkv[D + i];
    __syncwarp();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Fused step, context length 0: no attention, but the new token's k (rotated)
// and v still go into a valid slot, as kv_append would put them.  Run by the
// consumer threads of one CTA.
template <int D>
__device__ __noinline__ void append_only_e4m3(const DecodeParams& p, const RopeFreq& fr, int b) {
    constexpr int HALF = D / 2;
    const double pos = (double)p.positions[b];
    const int64_t slot = p.slot_mapping[b];
    const int64_t num_slots = (int64_t)p.num_blocks * kPageRows;
    if (slot >= num_slots && threadIdx.x == 0) report_error(p.err, PKV_DEVERR_SLOT);
    if (slot < 0 || slot >= num_slots) return;
    const uint16_t* kn = reinterpret_cast<const uint16_t*>(p.k_new) + (size_t)b * p.Hkv * D;
    const uint16_t* vn = reinterpret_cast<const uint16_t*>(p.v_new) + (size_t)b * p.Hkv * D;
    auto bf = [](uint16_t x) { return (double)__uint_as_float((uint32_t)x << 16); };
    const int64_t blk = slot / kPageRows;
    const int row = (int)(slot % kPageRows);
    for (int idx = threadIdx.x; idx < p.Hkv * HALF; idx += NW * 32) {
        const int h = idx / HALF, i = idx % HALF;
        uint8_t* pg = reinterpret_cast<uint8_t*>(p.k_cache) + (blk * p.Hkv + h) * (2 * kPageRows * D);
        double sn, cs, y0, y1;
        sincos(reduce_two_pi(pos * fr.f[i]), &sn, &cs);
        rope_rotate_f64(bf(kn[h * D + i]), bf(kn[h * D + i + HALF]), cs, sn, y0, y1);
        const uint32_t c = e4m3x2_scaled(y0, y1, (double)p.k_scale);
        pg[row * D + i] = (uint8_t)(c & 0xFFu);
        pg[row * D + i + HALF] = (uint8_t)(c >> 8);
    }
    for (int idx = threadIdx.x; idx < p.Hkv * D; idx += NW * 32) {
        const int h = idx / D, i = idx % D;
        uint8_t* pg = reinterpret_cast<uint8_t*>(p.k_cache) + (blk * p.Hkv + h) * (2 * kPageRows * D);
        pg[kPageRows * D + i * kPageRows + row] =
            (uint8_t)(e4m3x2_scaled(bf(vn[h * D + i]), 0.0, (double)p.v_scale) & 0xFFu);
    }
}

template <typename T, int D>
__device__ __noinline__ void append_only(const DecodeParams& p, const RopeFreq& fr, int b) {
    constexpr int HALF = D / 2;
    const double pos = (double)p.positions[b];
    const int64_t slot = p.slot_mapping[b];
    const int64_t num_slots = (int64_t)p.num_blocks * kPageRows;
    const bool write_kv = slot >= 0 && slot < num_slots;
    if (slot >= num_slots && threadIdx.x == 0) report_error(p.err, PKV_DEVERR_SLOT);
    const T* kn = reinterpret_cast<const T*>(p.k_new) + (size_t)b * p.Hkv * D;
    const T* vn = reinterpret_cast<const T*>(p.v_new) + (size_t)b * p.Hkv * D;
    const int64_t blk = write_kv ? slot / kPageRows : 0, row = write_kv ? slot % kPageRows : 0;
    const int nk = write_kv ? p.Hkv * HALF : 0;
    for (int idx = threadIdx.x; idx < nk; idx += NW * 32) {
        const int h = idx / HALF, i = idx % HALF;
        const T* src = kn + h * D;
        T* dst = reinterpret_cast<T*>(p.k_cache) + ((blk * p.Hkv + h) * kPageRows + row) * D;
        double sn, cs;
        sincos(reduce_two_pi(pos * fr.f[i]), &sn, &cs);
        const double x0 = to_d<T>(src[i]), x1 = to_d<T>(src[i + HALF]);
        dst[i] = from_d<T>(x0 * cs - x1 * sn);
        dst[i + HALF] = from_d<T>(x1 * cs + x0 * sn);
    }
    if (write_kv) {
        for (int idx = threadIdx.x; idx < p.Hkv * D; idx += NW * 32) {
            const int h = idx / D, i = idx % D;
            reinterpret_cast<T*>(p.v_cache)[((blk * p.Hkv + h) * kPageRows + row) * D + i] = vn[h * D + i];
        }
    }
}

// ---------------------------------------------------------------- producer

// Fused step, 8-bit cache: one warp makes the new token's codes of
// (sequence b, kv head h) exactly as the 8-bit append does (k rotated in
// fp64, x / scale in fp64 rounded to binary32, nearest E4M3), writes them
// into row `row` of the cache page `blk` and stages them at nk (k codes in
// [0, D), v codes in [D, 2D)) for the consumers' patch.
template <int D>
__device__ __forceinline__ void make_new_codes(const DecodeParams& p, int b, int h, double pos,
                                            const double (&f)[(D + 63) / 64], int row, int blk,
                                            uint8_t* nk) {
    constexpr int HALF = D / 2;
    const int lane = threadIdx.x & 31;
    const uint16_t* kn = reinterpret_cast<const uint16_t*>(p.k_new) + ((size_t)b * p.Hkv + h) * D;
    const uint16_t* vn = reinterpret_cast<const uint16_t*>(p.v_new) + ((size_t)b * p.Hkv + h) * D;
    uint8_t* gpage = reinterpret_cast<uint8_t*>(p.k_cache) +
                     ((size_t)blk * p.Hkv + h) * (size_t)(2 * kPageRows * D);
    auto bf = [](uint16_t x) { return (double)__uint_as_float((uint32_t)x << 16); };
#pragma unroll
    for (int u = 0; u < (D + 63) / 64; ++u) {
        const int i = lane + 32 * u;
        if (i < HALF) {
            double sn, cs, y0, y1;
            sincos(reduce_two_pi(pos * f[u]), &sn, &cs);
            rope_rotate_f64(bf(kn[i]), bf(kn[i + HALF]), cs, sn, y0, y1);
            const uint32_t c = e4m3x2_scaled(y0, y1, (double)p.k_scale);
            nk[i] = (uint8_t)(c & 0xFFu);
            nk[i + HALF] = (uint8_t)(c >> 8);
            gpage[row * D + i] = (uint8_t)(c & 0xFFu);
            gpage[row * D + i + HALF] = (uint8_t)(c >> 8);
        }
    }
    for (int i = lane; i < D; i += 32) {
        const uint8_t c = (uint8_t)(e4m3x2_scaled(bf(vn[i]), 0.0, (double)p.v_scale) & 0xFFu);
        nk[D + i] = c;
        gpage[kPageRows * D + i * kPageRows + row] = c;
    }
}


// Reads the producer issues before the context lengths are known, for the
// first item this CTA would get if every sequence had NP partitions (exact
// for uniform batches; a wrong guess costs the reads and nothing else).
template <int D>
struct FirstItemGuess {
    int b = -1, part = -1;
    int ent = -1;                 // block-table entry of page `lane` of the item
    int64_t slot = -1, pos = 0;   // fused step: the sequence's new token
    double f[(D + 63) / 64];      // fused step: RoPE frequencies of this lane
};

template <typename T, int D, int G, bool FUSED>
__device__ void run_producer(const DecodeParams& p, const FirstItemGuess<D>& guess,
                             const CUtensorMap* tmk, const CUtensorMap* tmv, uint8_t* base,
                             uint64_t* full, uint64_t* empty, uint64_t* qbar, uint32_t* masks,
                             volatile int* s_abort, const int* s_len, const int* s_pre, int W,
                             uint64_t* rank_bar, bool lpt) {
    using L = Layout<T, D, G>;
    const int lane = threadIdx.x & 31;
    int* s_item = reinterpret_cast<int*>(base + L::OFF_ITEM);
    // The longest-first order of the last partitions is ranked by the
    // consumer warps while this warp streams the full partitions, which come
    // first; before the first item that needs the order this warp waits for
    // it (false: the wait ran out).
    bool ranked = !lpt;
    const int nfull = s_pre[p.B];
    auto ensure_ranked = [&](int i) -> bool {
        if (ranked || i / p.Hkv < nfull) return true;
        int ok = 1;
        if (lane == 0) ok = mbar_wait(rank_bar, 0);
        ranked = __shfl_sync(0xffffffffu, ok, 0) != 0;
        return ranked;
    };

    // Work order of this CTA: items blockIdx.x and blockIdx.x + gridDim.x,
    // then items claimed one at a time from the counter (2 gridDim.x + its
    // old value), so that CTAs that finish early take more; without a
    // counter, blockIdx.x + k gridDim.x.  A claim is issued one item before
    // its result is needed, and nothing touches the returned value until
    // then (the warp would stall on it).  Claimed values only grow, so once
    // a CTA sees an item >= W every later claim is past W too and nothing
    // claimed is lost.
    int item = blockIdx.x;
    int item1 = item + (int)gridDim.x;  // the item after `item`
    if (p.cluster) {
        // cluster mode: CTA rank r of the cluster of (sequence, kv head) takes
        // partition r, if the sequence has one, and nothing else
        const int CS = p.cluster, cid = blockIdx.x / CS, rank = blockIdx.x - cid * CS;
        const int b = cid / p.Hkv, h = cid - b * p.Hkv;
        const int npb = (s_len[b] - window_page_start(p.window, s_len[b]) + p.P - 1) / p.P;
        item = rank < npb ? (s_pre[b] + rank) * p.Hkv + h : W;
        item1 = W;
    }
    uint32_t pend = 0;                  // lane 0: raw counter value of the claim in flight
    int k_static = 2;
    auto issue_claim = [&]() {
        if (p.sched && lane == 0) pend = atomicAdd(p.sched, 1u);
    };
    auto take_claim = [&]() -> int {
        int v;
        if (p.sched)
            v = 2 * (int)gridDim.x + (int)__shfl_sync(0xffffffffu, pend, 0);
        else
            v = (int)blockIdx.x + k_static * (int)gridDim.x;
        ++k_static;
        return v;
    };

    // Block-table entries are loaded a chunk ahead and range-checked only when
    // their chunk comes up: a check right after the load would stall the warp
    // on it (the error report is a side effect the compiler cannot defer).
    constexpr int kNoPage = INT_MIN;  // lane past the item's last page
    auto checked = [&](int v) -> int {
        if (v == kNoPage) return -1;
        if (v < 0 || v >= p.num_blocks) {
            report_error(p.err, PKV_DEVERR_BLOCK_ID);
            return -1;
        }
        return v;
    };
    auto raw_entry = [&](const Item& it, int page) -> int {
        if (page >= it.npages) return kNoPage;
        const int jb = it.t0 / kPageRows + page;
        return p.block_tables[(size_t)it.b * p.MB + jb];
    };

    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_parity[8];  // parity of the last issue into each stage
    uint32_t issued_any = 0;
    // qbar: per stage, the parity of its next phase and whether a q copy was issued
    uint32_t q_parity = 0, q_issued = 0;
    bool abort = false;
    if (item < W && !ensure_ranked(item)) {
        abort = true;
        item = W;
    }
    if (item < W) {
    if (item1 < W) issue_claim();
    Item cur = decode_item(item, p, s_len, s_pre);
    int c0 = 0;
    const bool hit = cur.b == guess.b && cur.part == guess.part;
    int cur_ent = hit ? (lane < cur.npages ? checked(guess.ent) : -1) : checked(raw_entry(cur, lane));
    // fused step: the new token's slot and position
    int64_t cur_slot = -1, cur_pos = 0;
    // fused step: the current item's rope table, computed ahead (for the
    // next item while this one's last stages are in flight)
    float rope_cs[(D + 63) / 64], rope_sn[(D + 63) / 64];
    if constexpr (FUSED) {
        cur_slot = hit ? guess.slot : p.slot_mapping[cur.b];
        cur_pos = hit ? guess.pos : p.positions[cur.b];
        warp_rope_regs<D>((double)cur_pos, guess.f, rope_cs, rope_sn);
    }
    int* patch = reinterpret_cast<int*>(base + L::OFF_PATCH);

    while (!abort) {
        // prefetch the block-table entries of the next chunk of 32 pages
        int nitem = item, nc0 = c0 + 32;
        Item nxt = cur;
        if (nc0 >= cur.npages) {
            nitem = item1;
            nc0 = 0;
            if (nitem < W) {
                if (ensure_ranked(nitem)) {
                    nxt = decode_item(nitem, p, s_len, s_pre);
                } else {
                    nitem = W;
                    abort = true;
                }
            }
        }
        const int nxt_raw = (nitem < W) ? raw_entry(nxt, nc0 + lane) : kNoPage;
        const bool new_item = FUSED && nitem != item && nitem < W;
        const int64_t nxt_slot = new_item ? p.slot_mapping[nxt.b] : cur_slot;
        const int64_t nxt_pos = new_item ? p.positions[nxt.b] : cur_pos;

        const int cend = min(cur.npages, c0 + 32);
        for (int s0 = c0; s0 < cend; s0 += L::STAGE_PAGES) {
            const int npg = min(L::STAGE_PAGES, cur.npages - s0);
            const int k = lane - (s0 - c0);
            const bool mine = k >= 0 && k < npg && cur_ent >= 0;
            const uint32_t vmask = __ballot_sync(0xffffffffu, mine) >> (s0 - c0);
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1) && !*s_abort;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                abort = true;
                break;
            }
            uint8_t* kdst = base + stage * L::STAGE_BYTES;
            uint8_t* vdst = kdst + L::VOFF;
            const bool first = (s0 == 0);
            // fused step: the sequence's last page gets the new token's row;
            // only when its slot is the one the block table gives that token
            int patch_row = -1, patch_blk = 0;
            if constexpr (FUSED) {
                if (s0 + L::STAGE_PAGES >= cur.npages && cur.part == cur.np - 1) {
                    const int lastpage = cur.npages - 1;
                    const int phys = __shfl_sync(0xffffffffu, cur_ent, lastpage - c0);
                    const int row = (s_len[cur.b] - 1) % kPageRows;
                    if (cur_slot >= 0) {
                        if (phys >= 0 && cur_slot == (int64_t)phys * kPageRows + row) {
                            patch_row = row;
                            patch_blk = phys;
                        } else if (lane == 0) {
                            report_error(p.err, PKV_DEVERR_SLOT);
                        }
                    }
                }
            }
            // The stage's bytes are announced first and the copies issued at
            // once; what the producer writes itself (mask, patch, rope table)
            // follows while the copies are in flight and is published by the
            // stage's one arrival.
            if (lane == 0) {
                const uint32_t bytes = __popc(vmask) * 2u * L::PAGE_BYTES +
                                       ((patch_row >= 0 && !L::F8) ? (uint32_t)L::NEWKV_BYTES : 0u);
                mbar_expect_tx(&full[stage], bytes);
            }
            __syncwarp();
            if (mine) {
                const int row0 = (cur_ent * p.Hkv + cur.h) * kPageRows;
                if constexpr (L::F8) {
                    // the page's [K | V] region: at d = 64 one box of 8 rows of
                    // 256 bytes; at d = 128 its K as 16 swizzled rows of 128
                    // bytes and its (transposed) V as 8 rows of 256 bytes
                    const int page = cur_ent * p.Hkv + cur.h;
                    if constexpr (D == 64) {
                        tma_load_2d(kdst + k * L::KPITCH, tmk, 0, page * 8, &full[stage]);
                    } else {
                        tma_load_2d(kdst + k * L::KPITCH, tmk, 0, page * 32, &full[stage]);
                        tma_load_2d(vdst + k * L::KPITCH, tmv, 0, page * 16 + 8, &full[stage]);
                    }
                } else {
#pragma unroll
                    for (int bx = 0; bx < L::BOXES; ++bx) {
                        tma_load_2d(kdst + k * L::KPITCH + bx * L::BOX_BYTES, tmk, bx * 64,
                                    row0, &full[stage]);
                        tma_load_2d(vdst + k * L::KPITCH + bx * L::BOX_BYTES, tmv, bx * 64,
                                    row0, &full[stage]);
                    }
                }
            }
            if (first && lane == 0) {
                const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q) +
                                      ((size_t)cur.b * p.Hq + (size_t)cur.h * G) * D * L::QSZ;
                mbar_expect_tx(&qbar[stage], L::Q_COPY);
                bulk_load(base + L::OFF_Q + stage * L::Q_BYTES, qsrc, L::Q_COPY, &qbar[stage]);
            }
            if constexpr (FUSED && L::F8) {
                // 8-bit cache: this warp makes the new token's codes exactly
                // as the 8-bit append does (k rotated in fp64, x / scale in
                // fp64 rounded to binary32, nearest E4M3), writes them to the
                // cache and stages them for the consumers' patch
                if (patch_row >= 0)
                    make_new_codes<D>(p, cur.b, cur.h, (double)cur_pos, guess.f, patch_row,
                                      patch_blk, base + L::OFF_NEWKV + stage * L::NEWKV_BYTES);
            } else if (FUSED && patch_row >= 0 && lane == 1) {
                const size_t row_off = ((size_t)cur.b * p.Hkv + cur.h) * L::ROW_COPY;
                uint8_t* nk = base + L::OFF_NEWKV + stage * L::NEWKV_BYTES;
                bulk_load(nk, reinterpret_cast<const uint8_t*>(p.k_new) + row_off, L::ROW_COPY,
                          &full[stage]);
                bulk_load(nk + L::ROW_COPY, reinterpret_cast<const uint8_t*>(p.v_new) + row_off,
                          L::ROW_COPY, &full[stage]);
            }
            if constexpr (FUSED) {
                // the rope table rides with the item's first stage (q) and,
                // for the bf16 / fp32 caches, with the stage that carries the
                // new token (its k)
                if (first || (!L::F8 && patch_row >= 0))
                    warp_rope_store<D>(rope_cs, rope_sn,
                                       reinterpret_cast<float*>(base + L::OFF_ROPE +
                                                                stage * L::ROPE_BYTES));
            }
            if (lane == 0) {
                masks[stage] = vmask;
                s_item[stage] = item;
                if constexpr (FUSED) {
                    patch[2 * stage] = patch_row;
                    patch[2 * stage + 1] = patch_blk;
                }
            }
            __syncwarp();
            if (lane == 0) {
                if (first) mbar_arrive(&qbar[stage]);
                mbar_arrive(&full[stage]);
            }
            issued_parity[stage] = phase;
            issued_any |= 1u << stage;
            if (first) {
                q_issued |= 1u << stage;
                q_parity ^= 1u << stage;
            }
            if (++stage == L::STAGES) {
                stage = 0;
                phase ^= 1;
            }
        }
        if (abort || nitem >= W) break;
        if (nitem != item) {
            item1 = take_claim();
            if (item1 < W) issue_claim();
            // the next item's table, while this item's stages are in flight
            if constexpr (FUSED) warp_rope_regs<D>((double)nxt_pos, guess.f, rope_cs, rope_sn);
        }
        item = nitem;
        c0 = nc0;
        cur = nxt;
        cur_ent = checked(nxt_raw);
        cur_slot = nxt_slot;
        cur_pos = nxt_pos;
    }
    }
    if (!abort && lane == 0) {
        // no more work: a stage without data whose item is -1 tells the consumers
        if (mbar_wait(&empty[stage], phase ^ 1) && !*s_abort) {
            s_item[stage] = -1;
            mbar_arrive(&qbar[stage]);
        } else {
            abort = true;
        }
    }
    abort = __shfl_sync(0xffffffffu, abort, 0);
    if (abort) {
        *s_abort = 1;
        if (lane == 0) {
            report_error(p.err, PKV_DEVERR_TIMEOUT);
            // let every copy this warp started land before the CTA can exit
            for (int s = 0; s < L::STAGES; ++s)
                if (issued_any & (1u << s)) (void)mbar_wait(&full[s], issued_parity[s]);
            for (int s = 0; s < L::STAGES; ++s)
                if (q_issued & (1u << s)) (void)mbar_wait(&qbar[s], ((q_parity >> s) & 1u) ^ 1u);
        }
        __syncwarp();
    }
    // This CTA has made its last claim.  The last CTA to get here puts both
    // counters back to zero for the next launch.
    if (p.sched && lane == 0) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
            atomicExch(p.sched, 0u);
            atomicExch(p.sched + 1, 0u);
        }
    }
}

// ------------------------------------------------------------ item merge

// Row g (head g of the item) of warp w's merge record in stage `st`.
template <typename T, int D, int G>
__device__ __forceinline__ float* merge_row(uint8_t* base, int st, int w, int g) {
    using L = Layout<T, D, G>;
    if constexpr (L::MERGE_SEPARATE)
        return reinterpret_cast<float*>(base + L::OFF_MERGE + (w * G + g) * L::MERGE_ROW_BYTES);
    uint8_t* kslot = base + st * L::STAGE_BYTES + w * L::PPW * L::KPITCH;
    // the 8-bit cache: the warp's pages are one region of 2 PPW pages
    uint8_t* row = (L::F8 || g < L::MERGE_ROWS_PER_SLOT)
                       ? kslot + g * L::MERGE_ROW_BYTES
                       : kslot + L::VOFF + (g - L::MERGE_ROWS_PER_SLOT) * L::MERGE_ROW_BYTES;
    return reinterpret_cast<float*>(row);
}

// Cluster mode: slot `r` of the landing area (local address; map it to rank 0
// for a remote store).
template <typename T, int D, int G>
__device__ __forceinline__ float* cluster_slot(const DecodeParams& p, uint8_t* base, int r) {
    using L = Layout<T, D, G>;
    return reinterpret_cast<float*>(base + L::land_offset(p.B) + r * L::CLUSTER_PART_BYTES);
}

// All consumer warps have written (o, m, l) per head into their merge rows
// of stage `st`; merge them and write the output row or the partition
// partial.
template <typename T, int D, int G>
__device__ __forceinline__ void merge_and_store(const DecodeParams& p, const Item& it,
                                                uint8_t* base, int st) {
    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
        const int g = idx / D, dim = idx - (idx / D) * D;
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, merge_row<T, D, G>(base, st, w, g)[D]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float* row = merge_row<T, D, G>(base, st, w, g);
            const float f = row[D] == kNegInf ? 0.f : fast_exp2(row[D] - M);
            num += f * row[dim];
            den += f * row[D + 1];
        }
        const size_t hq = (size_t)it.b * p.Hq + (size_t)it.h * G + g;
        // den == 0 only if every page of the item was rejected (bad block ids)
        float val = den > 0.f ? num / den : 0.f;
        if constexpr (Layout<T, D, G>::F8) val *= p.v_scale;
        if (p.cluster) {
            // cluster mode: this CTA's partial goes straight into its slot of
            // rank 0's landing area (distributed shared memory)
            const float* part = cluster_slot<T, D, G>(p, base, cluster_ctarank()) + g * (D + 2);
            st_dsmem_f32(dsmem_addr(part + dim, 0), val);
            if (dim == 0) {
                st_dsmem_f32(dsmem_addr(part + D, 0), M);
                st_dsmem_f32(dsmem_addr(part + D + 1, 0), den);
            }
        } else if (it.np == 1 && it.slot0 == 0) {
            store_out(p.out, hq * D + dim, val, p.out_bf16);
        } else {
            const size_t slot = hq * p.NP + it.slot0 + it.part;
            p.part_o[slot * D + dim] = val;
            if (dim == 0) {
                p.part_ml[slot * 2] = M;
                p.part_ml[slot * 2 + 1] = den;
            }
        }
    }
}

// Cluster mode, once every CTA of the cluster has stored its partial into its
// slot of rank 0's landing area (an empty one, m = -inf and l = 0, when it had
// no partition or gave up): one cluster barrier (release / acquire, so the
// remote stores are visible), then rank 0 merges the slots from its own
// shared memory and writes out[b, h*G .. h*G+G-1, :], the same log-sum-exp
// merge as the combine kernel.  The other CTAs leave after the barrier:
// nothing reads their shared memory.  Every thread of every CTA of the
// cluster calls this exactly once (it holds the cluster barrier).
template <typename T, int D, int G>
__device__ void cluster_merge(const DecodeParams& p, uint8_t* base) {
    cluster_sync_all();
    const int CS = p.cluster;
    if (cluster_ctarank() != 0 || threadIdx.x >= NW * 32) return;
    const int cid = blockIdx.x / CS;
    const int b = cid / p.Hkv, h = cid - (cid / p.Hkv) * p.Hkv;
    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
        const int g = idx / D, dim = idx - (idx / D) * D;
        float M = kNegInf;
        for (int r = 0; r < CS; ++r) M = fmaxf(M, cluster_slot<T, D, G>(p, base, r)[g * (D + 2) + D]);
        float num = 0.f, den = 0.f;
        for (int r = 0; r < CS; ++r) {
            const float* row = cluster_slot<T, D, G>(p, base, r) + g * (D + 2);
            const float m = row[D], l = row[D + 1];
            const float w = (m == kNegInf || l == 0.f) ? 0.f : l * fast_exp2(m - M);
            num = fmaf(w, row[dim], num);
            den += w;
        }
        const size_t hq = (size_t)b * p.Hq + (size_t)h * G + g;
        store_out(p.out, hq * D + dim, den > 0.f ? num / den : 0.f, p.out_bf16);
    }
}

// Bounded barrier of the consumer warps (every consumer thread arrives).
__device__ __forceinline__ bool consumer_sync(const DecodeParams& p, uint64_t* bar,
                                              uint32_t& phase, volatile int* s_abort) {
    mbar_arrive(bar);
    const bool ok = mbar_wait(bar, phase);
    phase ^= 1;
    if (!ok) {
        *s_abort = 1;
        report_error(p.err, PKV_DEVERR_TIMEOUT);
    }
    return ok;
}

// Fused step, page that holds the sequence's newest token: patch it in.
template <typename T, int D, int G, bool FUSED>
__device__ __forceinline__ void item_patch_page(const DecodeParams& p, const Item& it, int j,
                                                int slot, int stage, uint8_t* base) {
    if constexpr (FUSED) {
        using L = Layout<T, D, G>;
        // only the last page of a sequence's last partition can carry the
        // new token: test that (registers) before reading the stage's record
        if (j != it.npages - 1 || it.part != it.np - 1) return;
        const float* tab = reinterpret_cast<const float*>(base + L::OFF_ROPE + stage * L::ROPE_BYTES);
        const int* pt = reinterpret_cast<const int*>(base + L::OFF_PATCH) + 2 * stage;
        if constexpr (L::F8) {
            if (pt[0] >= 0) {
                uint8_t* kpage = base + stage * L::STAGE_BYTES + slot * L::KPITCH;
                patch_new_codes<D>(kpage, kpage + L::VOFF,
                                   base + L::OFF_NEWKV + stage * L::NEWKV_BYTES, pt[0]);
            }
            return;
        } else if (pt[0] >= 0) {
            const int row = pt[0];
            const size_t grow = (((size_t)pt[1] * p.Hkv + it.h) * kPageRows + row) * D;
            uint8_t* kpage = base + stage * L::STAGE_BYTES + slot * L::KPITCH;
            patch_new_row<T, D>(kpage, kpage + L::VOFF,
                                base + L::OFF_NEWKV + stage * L::NEWKV_BYTES, row, tab,
                                reinterpret_cast<T*>(p.k_cache) + grow,
                                reinterpret_cast<T*>(p.v_cache) + grow);
        }
    }
}

// ------------------------------------- tensor-core consumer (bf16, 8-bit cache)
//
// The 8-bit cache (T = e4m3kv) runs the same tiles as f16 MMAs: E4M3 codes
// widen to f16 exactly (cvt.rn.f16x2.e4m3x2), q is rounded to f16 (exact for
// bf16 values of magnitude 2^-17 .. 65504), and P is split into two f16
// terms.  Its fragments are read with plain shared-memory loads, in an
// order that lets each lane take whole 16-byte rows or 4-byte runs:
//   * scores: a lane's four k-values of k-step kk are the four consecutive
//     dims (D/4) cq + 4 kk .. +3 (the same order for q and K, so q.K is
//     unchanged), and lane row r of n-tile j reads token
//     pi(8j + r) = 2r - (r & 1) + 2j of the page, so that the score columns a
//     lane ends up with are the page's tokens 4 cq .. 4 cq + 3;
//   * output: those four tokens are the lane's k-values of the P V MMA, four
//     consecutive bytes of a transposed V row.

template <typename T, int D, int G, bool FUSED>
__device__ int run_consumer_mma(const DecodeParams& p, const RopeFreq& fr, uint8_t* base,
                                 uint64_t* full, uint64_t* empty, uint64_t* qbar,
                                 uint64_t* merge_bar,
                                 const uint32_t* masks, volatile int* s_abort, const int* s_len,
                                 const int* s_pre, int W) {
    using L = Layout<T, D, G>;
    constexpr bool F8 = L::F8;
    constexpr int KS = D / 16;  // k-steps of the score MMA
    constexpr int NT = D / 8;   // n-tiles of the output MMA
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, cq = lane & 3;
    // Which query head (and which part of the P split) this lane's A rows carry.
    //   G == 8: rows r (c0,c1) are the high part of head r, rows r+8 the low part.
    //   G <= 4: row r < G high part of head r, G <= r < 2G low part of head r-G.
    const int head_a = (G == 8) ? r : (r < 2 * G ? r % G : -1);  // head in A row r
    const int head_b = (G == 8) ? r : -1;                        // head in A row r+8
    const bool row_is_lo = (G < 8) && (r >= G) && (r < 2 * G);
    const bool row_used = (G == 8) || (r < 2 * G);

    int merged = 0;  // items merged (cluster mode: at most one)
    int stage = 0;
    uint32_t phase = 0, mphase = 0;
    uint32_t qph = 0;  // per stage, the parity of qbar's next phase
    // fused step: the item's rope table, staged by the producer with its first stage
    const float* tab = nullptr;

    const int* s_item = reinterpret_cast<const int*>(base + L::OFF_ITEM);
    for (;;) {
        // the item's first stage says on qbar which item it is (-1: no more
        // work); its q and rope table are there too, its pages come on full
        if (!mbar_wait(&qbar[stage], (qph >> stage) & 1u) || *s_abort) {
            *s_abort = 1;
            if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
            return -1;
        }
        qph ^= 1u << stage;
        const int item = s_item[stage];
        if (item < 0) return merged;
        const Item it = decode_item(item, p, s_len, s_pre);
        float o[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        float m_run = kNegInf, l_run = 0.f;
        uint32_t qa[KS][4];
        tab = reinterpret_cast<const float*>(base + L::OFF_ROPE + stage * L::ROPE_BYTES);
        const uint8_t* qs = base + L::OFF_Q + stage * L::Q_BYTES;
        if constexpr (FUSED) {
            // The staged q is the raw input.  The consumer threads rotate it
            // in place once (thread t takes the pairs t, t + 128, ...), each
            // element rounded to bf16 as the append would store it, and meet
            // before any fragment is read.  The rotated q never leaves shared
            // memory.
            constexpr int HALF = D / 2;
            bf16* qrow = reinterpret_cast<bf16*>(base + L::OFF_Q + stage * L::Q_BYTES);
            for (int idx = warp * 32 + lane; idx < G * HALF; idx += NW * 32) {
                const int g = idx / HALF, i = idx - g * HALF;
                bf16* row = qrow + g * D;
                const float x = __bfloat162float(row[i]), y = __bfloat162float(row[i + HALF]);
                const float c = tab[i], sn = tab[HALF + i];
                row[i] = __float2bfloat16_rn(fmaf(x, c, -y * sn));
                row[i + HALF] = __float2bfloat16_rn(fmaf(y, c, x * sn));
            }
            // the buffer's next writer is a bulk copy (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            if (!consumer_sync(p, merge_bar, mphase, s_abort)) return -1;
        }
        // A fragments of Q: rows = query heads (see head_a/head_b), cols = dims.
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            const int col = kk * 16 + 2 * cq;
            uint32_t a0 = 0, a1 = 0, a2 = 0, a3 = 0;
            if constexpr (F8) {
                // dims (D/4) cq + 4 kk .. +3 of the head, as two f16 pairs
                auto quad = [&](int head, uint32_t& lo, uint32_t& hi) {
                    const int c = (D / 4) * cq + 4 * kk;
                    const uint2 v = *reinterpret_cast<const uint2*>(qs + (head * D + c) * 2);
                    lo = pack_f16(bf16lo(v.x), bf16hi(v.x));
                    hi = pack_f16(bf16lo(v.y), bf16hi(v.y));
                };
                if (head_a >= 0) quad(head_a, a0, a2);
                if (head_b >= 0) quad(head_b, a1, a3);
            } else if (head_a >= 0) {
                const uint32_t* qr = reinterpret_cast<const uint32_t*>(qs + head_a * D * 2);
                a0 = qr[col / 2];
                a2 = qr[(col + 8) / 2];
            }
            if (!F8 && head_b >= 0) {
                const uint32_t* qr = reinterpret_cast<const uint32_t*>(qs + head_b * D * 2);
                a1 = qr[col / 2];
                a3 = qr[(col + 8) / 2];
            }
            qa[kk][0] = a0;  // row r,   cols col, col+1
            qa[kk][1] = a1;  // row r+8
            qa[kk][2] = a2;  // row r,   cols col+8, col+9
            qa[kk][3] = a3;  // row r+8
        }
        const int nst = (it.npages + L::STAGE_PAGES - 1) / L::STAGE_PAGES;
        bool ok = true;
        int last = stage;
        for (int s = 0; s < nst; ++s) {
            ok = mbar_wait(&full[stage], phase) && !*s_abort;
            if (!ok) break;
            // this warp's PPW consecutive pages of the stage (a page whose
            // block id was rejected counts as empty)
            constexpr int PPW = L::PPW;
            const int j0 = s * L::STAGE_PAGES + warp * PPW;
            const uint32_t mk = (masks[stage] >> (warp * PPW)) & ((1u << PPW) - 1u);
            if (j0 < it.npages && mk != 0u) {
                // tokens first[u] .. valid[u] - 1 of page u are attended (first > 0
                // only where a sliding window starts inside the page)
                int valid[PPW], first[PPW];
#pragma unroll
                for (int u = 0; u < PPW; ++u) {
                    const int jj = j0 + u;
                    valid[u] = (jj < it.npages && ((mk >> u) & 1u))
                                   ? min(kPageRows, it.t1 - (it.t0 + jj * kPageRows))
                                   : 0;
                    first[u] = max(0, it.lo - (it.t0 + jj * kPageRows));
                    if (valid[u] > 0)
                        item_patch_page<T, D, G, FUSED>(p, it, jj, warp * PPW + u, stage, base);
                }
                const uint32_t kbase =
                    smem_addr(base + stage * L::STAGE_BYTES + warp * PPW * L::KPITCH);
                const uint32_t vbase = kbase + L::VOFF;
                const int mi = lane >> 3, ri = lane & 7;

                // S^T tile: 16 rows (heads) x 16 PPW tokens, n-tiles of 8 tokens
                float sc[2 * PPW][4];
#pragma unroll
                for (int n = 0; n < 2 * PPW; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
                if constexpr (F8) {
                    // lane row r of n-tile j: token pi(8j + r) of the page, its
                    // bytes (D/4) cq .. (D/4)(cq + 1) - 1, one word per k-step
                    uint32_t kw[PPW][2][KS];
#pragma unroll
                    for (int u = 0; u < PPW; ++u)
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int tok = 2 * r - (r & 1) + 2 * j;
                            const uint32_t row = kbase + u * L::KPITCH + tok * D;
                            if constexpr (D == 64) {
                                ld_shared_v4(row + 16 * cq, kw[u][j][0], kw[u][j][1], kw[u][j][2],
                                             kw[u][j][3]);
                            } else {
                                // 128B swizzle: 16-byte chunk c of the row sits at c ^ (tok & 7)
                                ld_shared_v4(row + (((2 * cq) ^ (tok & 7)) << 4), kw[u][j][0],
                                             kw[u][j][1], kw[u][j][2], kw[u][j][3]);
                                ld_shared_v4(row + (((2 * cq + 1) ^ (tok & 7)) << 4), kw[u][j][4],
                                             kw[u][j][5], kw[u][j][6], kw[u][j][7]);
                            }
                        }
#pragma unroll
                    for (int kk = 0; kk < KS; ++kk)
#pragma unroll
                        for (int u = 0; u < PPW; ++u)
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                uint32_t b0, b1;
                                e4m3x4_to_f16x4(kw[u][j][kk], b0, b1);
                                mma_f16_16816(sc[2 * u + j], qa[kk], b0, b1);
                            }
                } else {
#pragma unroll
                    for (int kk = 0; kk < KS; ++kk) {
                        const int tok = ri + ((mi >> 1) << 3);
                        const int ch = 2 * kk + (mi & 1);
#pragma unroll
                        for (int u = 0; u < PPW; ++u) {
                            uint32_t b00, b01, b10, b11;
                            ldsm_x4(kbase + u * L::KPITCH + chunk_offset<bf16, D>(tok, ch), b00,
                                    b01, b10, b11);
                            mma_bf16_16816(sc[2 * u], qa[kk], b00, b01);
                            mma_bf16_16816(sc[2 * u + 1], qa[kk], b10, b11);
                        }
                    }
                }
                // online softmax in the log2 domain; rows r carry c0, c1
                float x[2 * PPW][2];
#pragma unroll
                for (int n = 0; n < 2 * PPW; ++n)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        // token of the page in this score register
                        const int tk = F8 ? 4 * cq + 2 * (n & 1) + e : (n & 1) * 8 + 2 * cq + e;
                        x[n][e] = (tk < valid[n >> 1] && tk >= first[n >> 1])
                                      ? sc[n][e] * p.scale_log2 : kNegInf;
                    }
                float mx = kNegInf;
#pragma unroll
                for (int n = 0; n < 2 * PPW; ++n) mx = fmaxf(mx, fmaxf(x[n][0], x[n][1]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_new = fmaxf(m_run, mx);
                const float alpha = fast_exp2(m_run - m_new);
                float pr[2 * PPW][2];
                float psum = 0.f;
#pragma unroll
                for (int n = 0; n < 2 * PPW; ++n) {
                    pr[n][0] = fast_exp2(x[n][0] - m_new);
                    pr[n][1] = fast_exp2(x[n][1] - m_new);
                    psum += pr[n][0] + pr[n][1];
                }
                l_run = l_run * alpha + psum;
                // alpha is exactly 1 in every row whose maximum did not grow;
                // skip the rescale when that holds for the whole warp
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
#pragma unroll
                for (int u = 0; u < PPW; ++u) {
                    // P of page u as the A operand of the output MMA: two-term bf16 split
                    uint32_t pa[4];
                    {
                        const float(&p0)[2] = pr[2 * u];
                        const float(&p1)[2] = pr[2 * u + 1];
                        uint32_t hi0, hi1, lo0, lo1;
                        if constexpr (F8) {
                            hi0 = pack_f16(p0[0], p0[1]);
                            hi1 = pack_f16(p1[0], p1[1]);
                            lo0 = pack_f16(p0[0] - f16lo(hi0), p0[1] - f16hi(hi0));
                            lo1 = pack_f16(p1[0] - f16lo(hi1), p1[1] - f16hi(hi1));
                        } else {
                            hi0 = pack_bf16(p0[0], p0[1]);
                            hi1 = pack_bf16(p1[0], p1[1]);
                            lo0 = pack_bf16(p0[0] - bf16lo(hi0), p0[1] - bf16hi(hi0));
                            lo1 = pack_bf16(p1[0] - bf16lo(hi1), p1[1] - bf16hi(hi1));
                        }
                        if (G == 8) {
                            pa[0] = hi0;
                            pa[1] = lo0;
                            pa[2] = hi1;
                            pa[3] = lo1;
                        } else {
                            pa[0] = row_used ? (row_is_lo ? lo0 : hi0) : 0u;
                            pa[2] = row_used ? (row_is_lo ? lo1 : hi1) : 0u;
                            pa[1] = 0u;
                            pa[3] = 0u;
                        }
                    }
                    // O += P V over the page's 16 tokens (rows past `valid` are zeroed:
                    // they may hold stale or never-written shared memory)
                    if constexpr (F8) {
                        // lane (r, cq), n-tile c: dim 8c + r, tokens 4cq .. 4cq + 3
                        uint32_t bm = 0xffffffffu;
                        if (valid[u] < kPageRows || first[u] > 0) {
                            bm = 0u;
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                if (4 * cq + e >= first[u] && 4 * cq + e < valid[u])
                                    bm |= 0xffu << (8 * e);
                        }
                        const uint32_t vrow = vbase + u * L::KPITCH + r * 16 + 4 * cq;
#pragma unroll
                        for (int c = 0; c < NT; ++c) {
                            uint32_t b0, b1;
                            e4m3x4_to_f16x4(ld_shared_u32(vrow + c * 128) & bm, b0, b1);
                            mma_f16_16816(o[c], pa, b0, b1);
                        }
                    } else {
                        uint32_t vmask_lo = 0xffffffffu, vmask_hi = 0xffffffffu;
                        if (valid[u] < kPageRows || first[u] > 0) {
                            const int k0 = 2 * cq, vu = valid[u], fu = first[u];
                            auto in = [&](int k) { return k >= fu && k < vu; };
                            vmask_lo = (in(k0) ? 0x0000ffffu : 0u) | (in(k0 + 1) ? 0xffff0000u : 0u);
                            vmask_hi = (in(k0 + 8) ? 0x0000ffffu : 0u) |
                                       (in(k0 + 9) ? 0xffff0000u : 0u);
                        }
#pragma unroll
                        for (int c = 0; c < NT; c += 2) {
                            const int tok = ri + ((mi & 1) << 3);
                            const int ch = c + (mi >> 1);
                            uint32_t v0, v1, v2, v3;
                            ldsm_x4_trans(vbase + u * L::KPITCH + chunk_offset<bf16, D>(tok, ch),
                                          v0, v1, v2, v3);
                            mma_bf16_16816(o[c], pa, v0 & vmask_lo, v1 & vmask_hi);
                            mma_bf16_16816(o[c + 1], pa, v2 & vmask_lo, v3 & vmask_hi);
                        }
                    }
                }
            }
            __syncwarp();
            // the item's last stage stays held: its page slots take the merge
            last = stage;
            if ((s + 1 < nst || L::MERGE_SEPARATE) && lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == L::STAGES) {
                stage = 0;
                phase ^= 1;
            }
        }
        if (!ok) {
            *s_abort = 1;
            if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
            return -1;
        }

        // per-warp result for each real head: add the low-part rows
        float of[NT][2];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            if (G == 8) {
                of[n][0] = o[n][0] + o[n][2];
                of[n][1] = o[n][1] + o[n][3];
            } else {
                of[n][0] = o[n][0] + __shfl_down_sync(0xffffffffu, o[n][0], 4 * G);
                of[n][1] = o[n][1] + __shfl_down_sync(0xffffffffu, o[n][1], 4 * G);
            }
        }
        float lsum = l_run;
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
        if (r < G) {
            float* row = merge_row<T, D, G>(base, last, warp, r);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                row[n * 8 + 2 * cq] = of[n][0];
                row[n * 8 + 2 * cq + 1] = of[n][1];
            }
            if (cq == 0) {
                row[D] = m_run;
                row[D + 1] = lsum;
            }
        }
        // the rows (generic-proxy writes) precede the TMA writes that refill
        // the stage after its release
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        // every consumer thread arrives once its rows are written; bounded wait
        mbar_arrive(merge_bar);
        if (!mbar_wait(merge_bar, mphase)) {
            *s_abort = 1;
            report_error(p.err, PKV_DEVERR_TIMEOUT);
            return -1;
        }
        mphase ^= 1;
        merge_and_store<T, D, G>(p, it, base, last);
        ++merged;
        __syncwarp();
        if constexpr (L::MERGE_SEPARATE) {
            // one merge region for all items: nobody writes the next item's
            // rows before every warp has read this item's
            if (!consumer_sync(p, merge_bar, mphase, s_abort)) return -1;
        } else {
            if (lane == 0) mbar_arrive(&empty[last]);
        }
    }
}

// ------------------------------------------------------- CUDA-core consumer

template <typename T, int D, int G, bool FUSED>
__device__ int run_consumer_simt(const DecodeParams& p, const RopeFreq& fr, uint8_t* base,
                                  uint64_t* full, uint64_t* empty, uint64_t* qbar,
                                  uint64_t* merge_bar,
                                  const uint32_t* masks, volatile int* s_abort, const int* s_len,
                                  const int* s_pre, int W) {
    using L = Layout<T, D, G>;
    constexpr bool IS_BF16 = std::is_same<T, bf16>::value;
    constexpr int EPL = 16 / (int)sizeof(T);  // elements per lane (one 16-byte chunk)
    constexpr int TPL = D / EPL;              // lanes per token row
    constexpr int TPW = 32 / TPL;             // tokens per warp pass
    constexpr int PASSES = kPageRows / TPW;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = lane % TPL, tg = lane / TPL;

    int merged = 0;  // items merged (cluster mode: at most one)
    int stage = 0;
    uint32_t phase = 0, mphase = 0;
    uint32_t qph = 0;  // per stage, the parity of qbar's next phase

    auto load16 = [&](uint32_t addr, float (&f)[EPL]) {
        uint32_t w0, w1, w2, w3;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                     : "r"(addr)
                     : "memory");
        if constexpr (IS_BF16) {
            f[0] = bf16lo(w0); f[1] = bf16hi(w0); f[2] = bf16lo(w1); f[3] = bf16hi(w1);
            f[4] = bf16lo(w2); f[5] = bf16hi(w2); f[6] = bf16lo(w3); f[7] = bf16hi(w3);
        } else {
            f[0] = __uint_as_float(w0); f[1] = __uint_as_float(w1);
            f[2] = __uint_as_float(w2); f[3] = __uint_as_float(w3);
        }
    };

    // fused step: the item's rope table, staged by the producer with its first stage
    const float* tab = nullptr;

    const int* s_item = reinterpret_cast<const int*>(base + L::OFF_ITEM);
    for (;;) {
        // the item's first stage says on qbar which item it is (-1: no more
        // work); its q and rope table are there too, its pages come on full
        if (!mbar_wait(&qbar[stage], (qph >> stage) & 1u) || *s_abort) {
            *s_abort = 1;
            if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
            return -1;
        }
        qph ^= 1u << stage;
        const int item = s_item[stage];
        if (item < 0) return merged;
        const Item it = decode_item(item, p, s_len, s_pre);
        float qf[G][EPL], o[G][EPL], m[G], l[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = kNegInf;
            l[g] = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[g][e] = 0.f;
        }
        tab = reinterpret_cast<const float*>(base + L::OFF_ROPE + stage * L::ROPE_BYTES);
        if constexpr (FUSED) {
            // raw q staged: rotate the lane's slice (rounded to T as an
            // appended q would be)
            const T* qrow0 = reinterpret_cast<const T*>(base + L::OFF_Q + stage * L::Q_BYTES);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < EPL; ++e)
                    qf[g][e] = (float)to_d<T>(from_f<T>(
                        rotated_elem<T, D>(qrow0 + g * D, c * EPL + e, tab)));
        } else {
            const uint32_t qs = smem_addr(base + L::OFF_Q + stage * L::Q_BYTES);
#pragma unroll
            for (int g = 0; g < G; ++g) load16(qs + g * D * (int)sizeof(T) + c * 16, qf[g]);
        }
        const int nst = (it.npages + L::STAGE_PAGES - 1) / L::STAGE_PAGES;
        bool ok = true;
        int last = stage;
        for (int s = 0; s < nst; ++s) {
            ok = mbar_wait(&full[stage], phase) && !*s_abort;
            if (!ok) break;
#pragma unroll 1
            for (int u = 0; u < L::PPW; ++u) {
            const int slot = warp * L::PPW + u;
            const int j = s * L::STAGE_PAGES + slot;
            if (j < it.npages && ((masks[stage] >> slot) & 1u)) {
                const int valid = min(kPageRows, it.t1 - (it.t0 + j * kPageRows));
                const int first = max(0, it.lo - (it.t0 + j * kPageRows));  // sliding window
                item_patch_page<T, D, G, FUSED>(p, it, j, slot, stage, base);
                const uint32_t kbase = smem_addr(base + stage * L::STAGE_BYTES + slot * L::KPITCH);
                const uint32_t vbase = kbase + L::VOFF;
#pragma unroll 2
                for (int ps = 0; ps < PASSES; ++ps) {
                    const int tk = ps * TPW + tg;
                    float kv[EPL];
                    load16(kbase + chunk_offset<T, D>(tk, c), kv);
                    float sdot[G];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < EPL; ++e) acc = fmaf(qf[g][e], kv[e], acc);
                        sdot[g] = acc;
                    }
#pragma unroll
                    for (int off = 1; off < TPL; off <<= 1)
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            sdot[g] += __shfl_xor_sync(0xffffffffu, sdot[g], off);
                    if (tk < valid && tk >= first) {
                        float vv[EPL];
                        load16(vbase + chunk_offset<T, D>(tk, c), vv);
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const float x = sdot[g] * p.scale_log2;
                            const float mn = fmaxf(m[g], x);
                            const float a = fast_exp2(m[g] - mn);
                            const float pe = fast_exp2(x - mn);
                            l[g] = l[g] * a + pe;
#pragma unroll
                            for (int e = 0; e < EPL; ++e) o[g][e] = fmaf(pe, vv[e], o[g][e] * a);
                            m[g] = mn;
                        }
                    }
                }
            }
            }
            __syncwarp();
            // the item's last stage stays held: its page slots take the merge
            last = stage;
            if ((s + 1 < nst || L::MERGE_SEPARATE) && lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == L::STAGES) {
                stage = 0;
                phase ^= 1;
            }
        }
        if (!ok) {
            *s_abort = 1;
            if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
            return -1;
        }
        // merge the token groups of this warp
#pragma unroll
        for (int off = TPL; off < 32; off <<= 1) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float m2 = __shfl_xor_sync(0xffffffffu, m[g], off);
                const float l2 = __shfl_xor_sync(0xffffffffu, l[g], off);
                const float M = fmaxf(m[g], m2);
                const float a = m[g] == kNegInf ? 0.f : fast_exp2(m[g] - M);
                const float a2 = m2 == kNegInf ? 0.f : fast_exp2(m2 - M);
                l[g] = l[g] * a + l2 * a2;
#pragma unroll
                for (int e = 0; e < EPL; ++e) {
                    const float o2 = __shfl_xor_sync(0xffffffffu, o[g][e], off);
                    o[g][e] = o[g][e] * a + o2 * a2;
                }
                m[g] = M;
            }
        }
        if (tg == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float* row = merge_row<T, D, G>(base, last, warp, g);
#pragma unroll
                for (int e = 0; e < EPL; ++e) row[c * EPL + e] = o[g][e];
                if (c == 0) {
                    row[D] = m[g];
                    row[D + 1] = l[g];
                }
            }
        }
        // the rows (generic-proxy writes) precede the TMA writes that refill
        // the stage after its release
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        // every consumer thread arrives once its rows are written; bounded wait
        mbar_arrive(merge_bar);
        if (!mbar_wait(merge_bar, mphase)) {
            *s_abort = 1;
            report_error(p.err, PKV_DEVERR_TIMEOUT);
            return -1;
        }
        mphase ^= 1;
        merge_and_store<T, D, G>(p, it, base, last);
        ++merged;
        __syncwarp();
        if constexpr (L::MERGE_SEPARATE) {
            // one merge region for all items: nobody writes the next item's
            // rows before every warp has read this item's
            if (!consumer_sync(p, merge_bar, mphase, s_abort)) return -1;
        } else {
            if (lane == 0) mbar_arrive(&empty[last]);
        }
    }
}

// ------------------------------------------------------------------ kernel

// Register budget: the d = 64 tensor-core kernels must fit three CTAs per SM
// (their shared-memory ring allows it), i.e. at most 128 registers a thread;
// the others run two CTAs per SM, which allows 168: ten warps spread over
// four SM sub-partitions put three on some, and 3 x 32 x 168 registers fit
// a sub-partition's 16384 (at 176 they would not, and only one CTA fits).
template <bool MMA, int D>
constexpr int decode_max_regs() { return (MMA && D == 64) ? 128 : 168; }

template <typename T, int D, int G, bool MMA, bool FUSED>
__global__ void __launch_bounds__(kDecodeThreads) __maxnreg__((decode_max_regs<MMA, D>()))
    paged_decode_kernel(const __grid_constant__ DecodeParams p,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ RopeFreq fr) {
    using L = Layout<T, D, G>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L::OFF_BAR);
    uint64_t* empty = full + L::STAGES;
    // an item's first stage publishes its q (and rope table) on qbar before
    // its pages complete full, so the q fragments are built while the
    // pages are still in flight
    uint64_t* qbar = empty + L::STAGES;
    uint64_t* merge_bar = qbar + L::STAGES;
    uint64_t* rank_bar = merge_bar + 1;
    uint32_t* masks = reinterpret_cast<uint32_t*>(base + L::OFF_MASK);
    int* misc = reinterpret_cast<int*>(base + L::OFF_MISC);
    volatile int* s_abort = misc;
    int* s_warp_tot = misc + 8;
    int* s_len = reinterpret_cast<int*>(base + L::OFF_SEQ);
    int* s_pre = s_len + p.B;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NW);
            mbar_init(&qbar[s], 1);
        }
        mbar_init(merge_bar, NW * 32);
        mbar_init(rank_bar, NW * 32);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == NW && lane == 0) {
        prefetch_tensor_map(&tm_k);
        prefetch_tensor_map(&tm_v);
    }

    // Everything below reads inputs a previous kernel may have written.
    grid_dependency_wait();
    grid_launch_dependents();

    // The producer starts the reads of its first item's block-table entries
    // (and, in the fused step, of the new token's slot and position) on a
    // guess, so that they overlap the scan of the context lengths below.
    FirstItemGuess<D> guess;
    if (warp == NW) {
        // every sequence at the maximum length: NP partitions each
        const int j = blockIdx.x / p.Hkv;
        int bs, ps;
        if (p.cluster) {
            const int cid = blockIdx.x / p.cluster;
            bs = cid / p.Hkv;
            ps = blockIdx.x - cid * p.cluster;
        } else if (p.B <= kLptMaxSeqs) {
            const int nf = p.NP - 1;  // full partitions per sequence, then the last ones
            if (j < p.B * nf) {
                bs = j / nf;
                ps = j - bs * nf;
            } else {
                bs = j - p.B * nf;
                ps = nf;
            }
        } else {
            bs = j / p.NP;
            ps = j - bs * p.NP;
        }
        if (bs < p.B && !p.shared_tokens && !p.window) {
            const int jb = ps * (p.P / kPageRows) + lane;
            guess.b = bs;
            guess.part = ps;
            guess.ent = jb < p.MB ? p.block_tables[(size_t)bs * p.MB + jb] : -1;
            if constexpr (FUSED) {
                guess.slot = p.slot_mapping[bs];
                guess.pos = p.positions[bs];
            }
        }
        if constexpr (FUSED) {
#pragma unroll
            for (int u = 0; u < (D + 63) / 64; ++u) guess.f[u] = fr.f[(lane + 32 * u) % 64];
        }
    }

    // Partition counts per sequence and their exclusive prefix (block scan);
    // in the longest-first order only the partitions before the last one.
    const int B = p.B;
    const bool lpt = B <= kLptMaxSeqs && !p.cluster && !p.shared_tokens;
    const int maxlen = p.MB * kPageRows;
    const int per = (B + kDecodeThreads - 1) / kDecodeThreads;
    const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
    int* s_rank = s_pre + B + 1;
    int* s_key = s_rank + B;
    int local = 0, local_ne = 0;
    for (int b = b0; b < b1; ++b) {
        int Lb = p.context_lens[b];
        if (Lb < 0 || Lb > maxlen) {
            report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
            Lb = Lb < 0 ? 0 : maxlen;
        }
        s_len[b] = Lb;
        int off = window_page_start(p.window, Lb);
        if (p.shared_tokens) {
            // cascade (at most kLptMaxSeqs sequences): whole pages, within the context
            int sh = p.shared_tokens[b];
            sh = sh < 0 ? 0 : (sh > Lb ? Lb : sh) / kPageRows * kPageRows;
            s_rank[b] = sh;
            off = max(off, sh);
        }
        const int npb = (Lb - off + p.P - 1) / p.P;
        const int cnt = lpt ? max(npb - 1, 0) : npb;
        if (lpt) s_key[b] = Lb > 0 ? (Lb - off) - (npb - 1) * p.P : -1;  // tokens of the last partition
        s_pre[b] = cnt;
        local += cnt;
        local_ne += Lb > 0;
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) s_warp_tot[warp] = incl;
    {
        const int ne_w = __reduce_add_sync(0xffffffffu, local_ne);
        if (lane == 0) misc[1 + warp] = ne_w;
    }
    __syncthreads();
    int run = incl - local;
    for (int w = 0; w < warp; ++w) run += s_warp_tot[w];
    for (int b = b0; b < b1; ++b) {
        const int cnt = s_pre[b];
        s_pre[b] = run;
        run += cnt;
    }
    if (tid == kDecodeThreads - 1) s_pre[B] = run;
    int ne = 0;  // contexts with tokens: one last partition each
    for (int w = 0; w <= NW; ++w) ne += misc[1 + w];
    __syncthreads();
    const int W = (s_pre[B] + (lpt ? ne : 0)) * p.Hkv;

    // In cluster mode no thread leaves before the cluster merge below.
    if (warp == NW) {
        run_producer<T, D, G, FUSED>(p, guess, &tm_k, &tm_v, base, full, empty, qbar, masks,
                                     s_abort, s_len, s_pre, W, rank_bar, lpt);
        if (!p.cluster) return;
    } else {
        if (lpt) {
            // rank of each last partition: longer first, then by sequence
            // (every CTA derives the same order); the producer is already
            // streaming the full partitions, which come first
            const int cper = (B + NW * 32 - 1) / (NW * 32);
            const int c0 = min(B, tid * cper), c1 = min(B, c0 + cper);
            for (int b = c0; b < c1; ++b) {
                const int k = s_key[b];
                if (k < 0) continue;
                int rank = 0;
                for (int b2 = 0; b2 < B; ++b2) {
                    const int k2 = s_key[b2];
                    rank += (k2 > k) || (k2 == k && b2 < b);
                }
                s_rank[rank] = b;
            }
            mbar_arrive(rank_bar);
            if (!mbar_wait(rank_bar, 0)) {
                *s_abort = 1;
                report_error(p.err, PKV_DEVERR_TIMEOUT);
            }
        }
        // zero the output of empty contexts (spread over the CTAs); in the
        // fused step their new token is still appended
        for (int b = blockIdx.x; b < B; b += gridDim.x) {
            if (s_len[b] != 0) continue;
            for (int idx = tid; idx < p.Hq * D; idx += NW * 32)
                store_out(p.out, (size_t)b * p.Hq * D + idx, 0.f, p.out_bf16);
            if constexpr (FUSED) {
                if constexpr (L::F8) append_only_e4m3<D>(p, fr, b);
                else append_only<T, D>(p, fr, b);
            }
        }
        int merged;
        if constexpr (MMA) {
            merged = run_consumer_mma<T, D, G, FUSED>(p, fr, base, full, empty, qbar, merge_bar, masks,
                                                      s_abort, s_len, s_pre, W);
        } else {
            merged = run_consumer_simt<T, D, G, FUSED>(p, fr, base, full, empty, qbar, merge_bar, masks,
                                                       s_abort, s_len, s_pre, W);
        }
        if (p.cluster && merged <= 0) {
            // no partition here (or this CTA gave up): an empty partial
            const float* part = cluster_slot<T, D, G>(p, base, cluster_ctarank());
            for (int idx = tid; idx < G * (D + 2); idx += NW * 32)
                st_dsmem_f32(dsmem_addr(part + idx, 0), (idx % (D + 2)) == D ? kNegInf : 0.f);
        }
    }
    if (p.cluster) cluster_merge<T, D, G>(p, base);
}

// ----------------------------------------------------------------- combine

struct CombineParams {
    const int32_t* context_lens;
    const int32_t* shared_tokens;  // cascade: slot 0 holds the shared-prefix partial
    int window;                    // sliding window (partitions start at its page)
    const float* part_o;
    const float* part_ml;
    void* out;
    int Hq, MB, P, NP;
    int out_bf16;
};

// out[b, h*G+g, :] = sum_p w_p o_p with w_p = l_p 2^(m_p - M) / sum_q l_q 2^(m_q - M),
// the exact log-sum-exp merge of the partition partials.  One CTA per
// (kv head, sequence); written for latency, since it sits at the end of every
// split decode:
//   * the context length and the (m, l) pairs of all NP possible partitions
//     are loaded together (pairs past the sequence's own count are ignored);
//   * every thread owns one float4 column chunk of one partition group and
//     loads its first partials before the weights are known;
//   * all heads' column sums meet in shared memory once, then are reduced.
// Threads per combine CTA: one warp per head for the weights, four warps at
// least.  At 128 threads (G <= 4) the ragged batch's 512 CTAs are resident at
// once (at 256 threads and 80 registers three fit an SM, and 68 CTAs waited
// for the first ones to leave).
template <int G>
constexpr int combine_threads() { return G <= 4 ? 128 : 32 * G; }

template <int D, int G>
__global__ void __launch_bounds__(combine_threads<G>()) combine_kernel(const __grid_constant__ CombineParams p) {
    constexpr int kCombineThreads = combine_threads<G>();
    constexpr int CH = D / 4;                   // float4 chunks per row
    constexpr int PG = kCombineThreads / CH;    // partition groups
    constexpr int kCombineUnroll = G >= 8 ? 1 : 8 / G;  // partitions in flight per head
    extern __shared__ float4 smem4[];
    float4* red = smem4;                                        // [G][PG][CH]
    float* w = reinterpret_cast<float*>(smem4 + G * PG * CH);   // [G][NP]
    grid_dependency_wait();
    const int b = blockIdx.y, h = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t hq0 = (size_t)b * p.Hq + (size_t)h * G;
    const int maxlen = p.MB * kPageRows;
    int Lb = p.context_lens[b];
    // (m, l) of this warp's head, all NP slots, issued with the length load
    constexpr int MLR = 8;                      // slots per lane kept in registers
    float2 ml[MLR];
    const int g_w = warp;                       // warps 0..G-1 own one head each
    if (g_w < G) {
        const float2* src = reinterpret_cast<const float2*>(p.part_ml + (hq0 + g_w) * p.NP * 2);
#pragma unroll
        for (int r = 0; r < MLR; ++r) {
            const int k = lane + 32 * r;
            ml[r] = k < p.NP ? src[k] : make_float2(kNegInf, 0.f);
        }
    }
    Lb = Lb < 0 ? 0 : (Lb > maxlen ? maxlen : Lb);
    int off = 0;
    const int woff = window_page_start(p.window, Lb);
    if (p.shared_tokens) {
        off = p.shared_tokens[b];
        off = off < 0 ? 0 : (off > Lb ? Lb : off) / kPageRows * kPageRows;
    }
    // slots: the shared prefix (cascade, when it has tokens), then the
    // partitions, from the later of the prefix's end and the window's page
    const int np = (off > 0 ? 1 : 0) + (Lb - max(off, woff) + p.P - 1) / p.P;
    if (np <= 1 && off == 0) return;  // written by the decode kernel

    // first partials of this thread, independent of the weights
    const int ch = threadIdx.x % CH, pg = threadIdx.x / CH;
    float4 v0[G][kCombineUnroll];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int u = 0; u < kCombineUnroll; ++u) {
            const int k = pg + u * PG;
            v0[g][u] = k < np ? reinterpret_cast<const float4*>(
                                    p.part_o + ((hq0 + g) * p.NP + k) * D)[ch]
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        }

    // weights: warp g turns head g's (m, l) pairs into normalised weights
    if (g_w < G) {
        const float2* src = reinterpret_cast<const float2*>(p.part_ml + (hq0 + g_w) * p.NP * 2);
        float M = kNegInf;
#pragma unroll
        for (int r = 0; r < MLR; ++r)
            if (lane + 32 * r < np) M = fmaxf(M, ml[r].x);
        for (int k = lane + 32 * MLR; k < np; k += 32) M = fmaxf(M, src[k].x);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float S = 0.f;
        float e[MLR];
#pragma unroll
        for (int r = 0; r < MLR; ++r) {
            const int k = lane + 32 * r;
            e[r] = (k < np && ml[r].x != kNegInf) ? fast_exp2(ml[r].x - M) * ml[r].y : 0.f;
            S += e[r];
        }
        for (int k = lane + 32 * MLR; k < np; k += 32) {
            const float2 v = src[k];
            const float ek = v.x == kNegInf ? 0.f : fast_exp2(v.x - M) * v.y;
            w[g_w * p.NP + k] = ek;
            S += ek;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) S += __shfl_xor_sync(0xffffffffu, S, off);
        const float inv = S > 0.f ? 1.f / S : 0.f;
#pragma unroll
        for (int r = 0; r < MLR; ++r) {
            const int k = lane + 32 * r;
            if (k < np) w[g_w * p.NP + k] = e[r] * inv;
        }
        for (int k = lane + 32 * MLR; k < np; k += 32) w[g_w * p.NP + k] *= inv;
    }
    __syncthreads();

    float4 acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        acc[g] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < kCombineUnroll; ++u) {
            const int k = pg + u * PG;
            const float wk = k < np ? w[g * p.NP + k] : 0.f;
            acc[g].x = fmaf(wk, v0[g][u].x, acc[g].x);
            acc[g].y = fmaf(wk, v0[g][u].y, acc[g].y);
            acc[g].z = fmaf(wk, v0[g][u].z, acc[g].z);
            acc[g].w = fmaf(wk, v0[g][u].w, acc[g].w);
        }
    }
    // partitions beyond the first kCombineUnroll rounds (long contexts)
#pragma unroll 2
    for (int k = pg + kCombineUnroll * PG; k < np; k += PG) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float4 v = reinterpret_cast<const float4*>(p.part_o + ((hq0 + g) * p.NP + k) * D)[ch];
            const float wk = w[g * p.NP + k];
            acc[g].x = fmaf(wk, v.x, acc[g].x);
            acc[g].y = fmaf(wk, v.y, acc[g].y);
            acc[g].z = fmaf(wk, v.z, acc[g].z);
            acc[g].w = fmaf(wk, v.w, acc[g].w);
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) red[(g * PG + pg) * CH + ch] = acc[g];
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * CH; idx += kCombineThreads) {
        const int g = idx / CH, c = idx - (idx / CH) * CH;
        float4 sum = red[(g * PG) * CH + c];
        for (int q = 1; q < PG; ++q) {
            const float4 v = red[(g * PG + q) * CH + c];
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
        }
        const size_t o = (hq0 + g) * D + c * 4;
        store_out(p.out, o, sum.x, p.out_bf16);
        store_out(p.out, o + 1, sum.y, p.out_bf16);
        store_out(p.out, o + 2, sum.z, p.out_bf16);
        store_out(p.out, o + 3, sum.w, p.out_bf16);
    }
    // the next launch (the next step's decode) starts once every CTA of this
    // grid is done or here (a CTA that returned early counts as done), so
    // that its CTAs find the SMs free; its own wait still orders it after
    // this grid's writes
    grid_launch_dependents();
}

// ------------------------------------------------------------------- host

int current_device() {
    int dev = 0;
    cudaGetDevice(&dev);
    return dev;
}

// Cluster-mode launches ask for this much shared memory per CTA, so that a
// cluster spreads over one SM per CTA instead of packing three CTAs into an
// SM (they share its issue slots and load bandwidth otherwise).
constexpr size_t kClusterCtaSmem = 116 * 1024;

template <typename K>
cudaError_t prepare_kernel(K kern, size_t smem, int* ctas_per_sm) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, size_t>, int> cache;
    const int dev = current_device();
    const auto key = std::make_tuple(reinterpret_cast<const void*>(kern), dev, smem);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
        *ctas_per_sm = it->second;
        return cudaSuccess;
    }
    // allow up to the device's opt-in maximum: cluster-mode launches ask for
    // more than the layout (spreading, plus the landing area of rank 0)
    int optin = 0;
    cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    if ((size_t)optin < smem) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kDecodeThreads, smem);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    cache[key] = n;
    *ctas_per_sm = n;
    return cudaSuccess;
}

// Clusters of `cs` CTAs of this kernel that can be resident at once (cached).
template <typename K>
cudaError_t max_active_clusters(K kern, size_t smem, int cs, int* n) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, size_t, int>, int> cache;
    const int dev = current_device();
    const auto key = std::make_tuple(reinterpret_cast<const void*>(kern), dev, smem, cs);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
        *n = it->second;
        return cudaSuccess;
    }
    cudaError_t e = cudaSuccess;
    if (cs > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cs);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int c = 0;
    e = cudaOccupancyMaxActiveClusters(&c, kern, &cfg);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();  // not fatal: no cluster mode for this shape
        c = 0;
    }
    cache[key] = c;
    *n = c;
    return cudaSuccess;
}

template <typename T, int D, int G, bool MMA, bool FUSED>
cudaError_t launch_decode_typed(const DecodeArgs& a, const CUtensorMap& tmk,
                                const CUtensorMap& tmv) {
    using L = Layout<T, D, G>;
    auto kern = paged_decode_kernel<T, D, G, MMA, FUSED>;
    const size_t smem = L::smem_bytes((int)a.B);
    int occ = 0;
    cudaError_t e = prepare_kernel(kern, smem, &occ);
    if (e != cudaSuccess) return e;

    DecodeParams p;
    p.q = a.q;
    p.block_tables = a.block_tables;
    p.context_lens = a.context_lens;
    p.out = a.out;
    p.part_o = a.part_o;
    p.part_ml = a.part_ml;
    p.sched = a.sched;
    p.shared_tokens = a.shared_tokens;
    p.window = a.window;
    p.err = a.device_error;
    p.B = (int)a.B;
    p.Hq = (int)a.Hq;
    p.Hkv = (int)a.Hkv;
    p.MB = (int)a.MB;
    p.P = a.partition_tokens;
    p.NP = a.max_partitions;
    p.num_blocks = (int)a.num_blocks;
    p.scale_log2 = a.scale * 1.4426950408889634f * (L::F8 ? a.k_scale : 1.0f);
    p.v_scale = L::F8 ? a.v_scale : 1.0f;
    p.k_scale = L::F8 ? a.k_scale : 1.0f;
    p.out_bf16 = a.out_dtype == PKV_DTYPE_BF16;
    p.k_new = a.k_new;
    p.v_new = a.v_new;
    p.positions = a.positions;
    p.slot_mapping = a.slot_mapping;
    p.k_cache = const_cast<void*>(a.k_cache);
    p.v_cache = const_cast<void*>(a.v_cache);
    RopeFreq fr;
    for (int i = 0; i < 64; ++i) fr.f[i] = (FUSED && i < D / 2) ? std::pow(a.theta, -(2.0 * i) / D) : 0.0;

    const int64_t upper = a.B * a.Hkv * (int64_t)a.max_partitions;
    const int64_t resident = (int64_t)device_sm_count() * occ;
    unsigned grid = (unsigned)std::max<int64_t>(1, std::min(upper, resident));

    // Cluster mode: when every (sequence, kv head) can have its own cluster of
    // NP CTAs resident at once, the partitions are merged inside the cluster
    // and the combine kernel is not needed.
    int cs = 0;
    const size_t smem_cl =
        std::max(L::cluster_smem_bytes((int)a.B, std::max(2, a.max_partitions)), kClusterCtaSmem);
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, current_device());
    if (e != cudaSuccess) return e;
    if (a.allow_cluster && !a.shared_tokens && a.max_partitions >= 2 &&
        a.max_partitions <= kMaxClusterCtas && smem_cl <= (size_t)optin) {
        int nc = 0;
        e = max_active_clusters(kern, smem_cl, a.max_partitions, &nc);
        if (e != cudaSuccess) return e;
        if ((int64_t)nc >= a.B * a.Hkv) cs = a.max_partitions;
    }
    p.cluster = cs;
    if (a.plan_only) {
        *a.launches = (cs || a.max_partitions <= 1) ? 1 : 2;
        return cudaSuccess;
    }
    if (cs) {
        p.sched = nullptr;  // one item per CTA, nothing to claim
        grid = (unsigned)(a.B * a.Hkv * cs);
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = cs ? smem_cl : smem;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)(cs ? cs : 1);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cs ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, p, tmk, tmv, fr);
    if (e != cudaSuccess || a.max_partitions <= 1 || cs) return e;
    if (a.launch_between) {
        e = a.launch_between(a.between_ctx);
        if (e != cudaSuccess) return e;
    }

    CombineParams cp;
    cp.context_lens = a.context_lens;
    cp.part_o = a.part_o;
    cp.part_ml = a.part_ml;
    cp.out = a.out;
    cp.Hq = (int)a.Hq;
    cp.MB = (int)a.MB;
    cp.P = a.partition_tokens;
    cp.NP = a.max_partitions;
    cp.out_bf16 = p.out_bf16;
    cp.shared_tokens = a.shared_tokens;
    cp.window = a.window;
    auto ckern = combine_kernel<D, G>;
    {
        static std::mutex mu;
        static size_t set_bytes[64] = {0};
        const int dev = current_device();
        std::lock_guard<std::mutex> lock(mu);
        if (dev >= 0 && dev < 64 && set_bytes[dev] < (size_t)(G * combine_threads<G>() * 16 + G * kMaxPartitions * 4)) {
            e = cudaFuncSetAttribute(ckern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     G * combine_threads<G>() * 16 + G * kMaxPartitions * 4);
            if (e != cudaSuccess) return e;
            set_bytes[dev] = (size_t)(G * combine_threads<G>() * 16 + G * kMaxPartitions * 4);
        }
    }
    const size_t csmem = (size_t)G * combine_threads<G>() * 16 + (size_t)G * a.max_partitions * sizeof(float);
    cudaLaunchConfig_t cc = cfg;
    cc.gridDim = dim3((unsigned)a.Hkv, (unsigned)a.B);
    cc.blockDim = dim3(combine_threads<G>());
    cc.dynamicSmemBytes = csmem;
    return cudaLaunchKernelEx(&cc, ckern, cp);
}

template <typename T, int D, bool MMA, bool FUSED>
cudaError_t dispatch_g(const DecodeArgs& a, const CUtensorMap& k, const CUtensorMap& v) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_decode_typed<T, D, 1, MMA, FUSED>(a, k, v);
        case 2: return launch_decode_typed<T, D, 2, MMA, FUSED>(a, k, v);
        case 4: return launch_decode_typed<T, D, 4, MMA, FUSED>(a, k, v);
        case 8: return launch_decode_typed<T, D, 8, MMA, FUSED>(a, k, v);
    }
    return cudaErrorInvalidValue;
}

template <bool FUSED>
cudaError_t dispatch_all(const DecodeArgs& a, const CUtensorMap& tmk, const CUtensorMap& tmv) {
    if (a.kv_dtype == PKV_DTYPE_E4M3) {
        return a.D == 64 ? dispatch_g<e4m3kv, 64, true, FUSED>(a, tmk, tmv)
                         : dispatch_g<e4m3kv, 128, true, FUSED>(a, tmk, tmv);
    }
    if (a.kv_dtype == PKV_DTYPE_F32) {
        return a.D == 64 ? dispatch_g<float, 64, false, FUSED>(a, tmk, tmv)
                         : dispatch_g<float, 128, false, FUSED>(a, tmk, tmv);
    }
    if (a.force_simt) {
        return a.D == 64 ? dispatch_g<bf16, 64, false, FUSED>(a, tmk, tmv)
                         : dispatch_g<bf16, 128, false, FUSED>(a, tmk, tmv);
    }
    return a.D == 64 ? dispatch_g<bf16, 64, true, FUSED>(a, tmk, tmv)
                     : dispatch_g<bf16, 128, true, FUSED>(a, tmk, tmv);
}

}  // namespace

cudaError_t encode_cache_map(CUtensorMap* map, const void* cache, int64_t num_blocks, int64_t Hkv,
                             int64_t D, int32_t dtype);
cudaError_t encode_vt_cache_map(CUtensorMap* map, const void* cache, int64_t num_blocks,
                                int64_t Hkv, int64_t D);

cudaError_t launch_paged_decode(const DecodeArgs& a) {
    CUtensorMap tmk, tmv;
    if (a.plan_only) {
        memset(&tmk, 0, sizeof(tmk));
        memset(&tmv, 0, sizeof(tmv));
        return a.fused ? dispatch_all<true>(a, tmk, tmv) : dispatch_all<false>(a, tmk, tmv);
    }
    cudaError_t e = encode_cache_map(&tmk, a.k_cache, a.num_blocks, a.Hkv, a.D, a.kv_dtype);
    if (e != cudaSuccess) return e;
    e = a.kv_dtype == PKV_DTYPE_E4M3 ? encode_vt_cache_map(&tmv, a.v_cache, a.num_blocks, a.Hkv, a.D)
                                     : encode_cache_map(&tmv, a.v_cache, a.num_blocks, a.Hkv, a.D,
                                                        a.kv_dtype);
    if (e != cudaSuccess) return e;
    return a.fused ? dispatch_all<true>(a, tmk, tmv) : dispatch_all<false>(a, tmk, tmv);
}

int decode_cluster_capacity(int cs) {
    // Every decode variant runs at one CTA per SM in cluster mode (its
    // shared-memory request sees to that), so one variant stands for all.
    auto kern = paged_decode_kernel<bf16, 64, 4, true, false>;
    int occ = 0, n = 0;
    if (prepare_kernel(kern, kClusterCtaSmem, &occ) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    if (max_active_clusters(kern, kClusterCtaSmem, cs, &n) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    return n;
}

int decode_ctas_per_sm(int64_t D, int64_t G, int32_t kv_dtype, bool simt, int64_t num_seqs) {
    // Estimate from the shared-memory footprint (the occupancy query needs a
    // device; this is used for host-side planning only).
    size_t smem = 0;
    const int B = (int)num_seqs;
    auto pick = [&](auto tag) { smem = decltype(tag)::smem_bytes(B); };
    auto by_g = [&](auto t, auto d) {
        using T = decltype(t);
        constexpr int Dv = decltype(d)::value;
        if (G <= 1) pick(Layout<T, Dv, 1>{});
        else if (G == 2) pick(Layout<T, Dv, 2>{});
        else if (G == 4) pick(Layout<T, Dv, 4>{});
        else pick(Layout<T, Dv, 8>{});
    };
    if (kv_dtype == PKV_DTYPE_F32) {
        if (D == 64) by_g(float{}, std::integral_constant<int, 64>{});
        else by_g(float{}, std::integral_constant<int, 128>{});
    } else if (kv_dtype == PKV_DTYPE_E4M3) {
        if (D == 64) by_g(e4m3kv{}, std::integral_constant<int, 64>{});
        else by_g(e4m3kv{}, std::integral_constant<int, 128>{});
    } else {
        if (D == 64) by_g(bf16{}, std::integral_constant<int, 64>{});
        else by_g(bf16{}, std::integral_constant<int, 128>{});
    }
    (void)simt;
    const size_t per_sm = 228 * 1024;
    int n = (int)(per_sm / (smem + 1024));
    return std::max(1, std::min(n, 3));
}

}  // namespace pkv
