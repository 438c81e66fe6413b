// pkv_api.cu -- the library's C ABI: argument validation, launch planning
// (partition length, workspace layout), TMA descriptor encoding, and error
// reporting.  No entry point allocates device memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "pkv_internal.h"

namespace pkv {

namespace {
thread_local char g_last_error[512] = "";

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
}  // namespace

void set_last_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
}

int device_sm_count() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// ---- TMA descriptors -------------------------------------------------------

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}
}  // namespace

// The cache [num_blocks, Hkv, 16, D] viewed as a 2-D tensor of num_blocks*Hkv*16
// rows of D elements; one box is one 16-row page (bf16: 64 columns per box,
// 128-byte swizzle; fp32: the whole row, no swizzle).
//
// The 8-bit cache is [num_blocks, Hkv, 2, 16 D] bytes: per page its K codes
// [16][D], then its V codes transposed [D][16].  At D = 64 the page's 2 KiB
// are one box of 8 rows of 256 bytes (the same bytes in the same order in
// shared memory, one request per page).  At D = 128 this map covers the
// cache as rows of 128 bytes (32 per page) and one box is the page's K half,
// 16 rows, 128-byte swizzled; encode_vt_cache_map gives its V half.
cudaError_t encode_cache_map(CUtensorMap* map, const void* cache, int64_t num_blocks, int64_t Hkv,
                             int64_t D, int32_t dtype) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const bool bf = dtype == PKV_DTYPE_BF16;
    const bool f8 = dtype == PKV_DTYPE_E4M3;
    const int esz = f8 ? 1 : (bf ? 2 : 4);
    const int row_bytes = f8 ? (D == 64 ? 256 : 128) : (int)(D * esz);
    const int rows_per_page = f8 ? (D == 64 ? 8 : 32) : kPageRows;
    const int box_rows = f8 ? (D == 64 ? 8 : kPageRows) : kPageRows;
    const cuuint64_t rows = (cuuint64_t)(num_blocks * Hkv * rows_per_page);
    cuuint64_t dims[2] = {(cuuint64_t)(row_bytes / esz), rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)(bf ? 64 : row_bytes / esz), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    // bf16 boxes are 128-byte rows, swizzled; 8-bit rows of 128 bytes too
    const bool swz = bf || (f8 && D == 128);
    CUresult r = fn(map,
                    f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                       : (bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32),
                    2, const_cast<void*>(cache), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The 8-bit cache at D = 128 as rows of 256 bytes (16 per page); one box is a
// page's V half, its transposed V codes [128][16] as 8 rows of 256 bytes
// (page p's V half starts at row 16 p + 8).
cudaError_t encode_vt_cache_map(CUtensorMap* map, const void* cache, int64_t num_blocks,
                                int64_t Hkv, int64_t D) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {256, (cuuint64_t)(num_blocks * Hkv * (2 * kPageRows * D / 256))};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {256, (cuuint32_t)(kPageRows * D / 256)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(cache), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// ---- shared validation -----------------------------------------------------

namespace {
pkv_status check_heads(int64_t Hq, int64_t Hkv, int64_t D, int64_t bs) {
    if (Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0) {
        set_last_error("head counts, head_dim and block_size must be positive");
        return PKV_ERR_INVALID_ARG;
    }
    if (Hq % Hkv != 0) {
        set_last_error("num_q_heads (%lld) is not a multiple of num_kv_heads (%lld)",
                       (long long)Hq, (long long)Hkv);
        return PKV_ERR_INVALID_ARG;
    }
    const int64_t G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) {
        set_last_error("group size Hq/Hkv = %lld not in {1, 2, 4, 8}", (long long)G);
        return PKV_ERR_UNSUPPORTED;
    }
    if (D != 64 && D != 128) {
        set_last_error("head_dim %lld not in {64, 128}", (long long)D);
        return PKV_ERR_UNSUPPORTED;
    }
    if (bs != kPageRows) {
        set_last_error("block_size %lld unsupported (16 only)", (long long)bs);
        return PKV_ERR_UNSUPPORTED;
    }
    if (Hkv > 256 || Hq > 2048) {
        set_last_error("too many heads");
        return PKV_ERR_UNSUPPORTED;
    }
    return PKV_OK;
}

bool valid_dtype(int32_t t) { return t == PKV_DTYPE_F32 || t == PKV_DTYPE_BF16; }
// Cache dtypes the planning calls accept (the 8-bit cache included).
bool valid_kv_dtype(int32_t t) { return valid_dtype(t) || t == PKV_DTYPE_E4M3; }

// Partition length.  A partition should fill whole stages of the ring and be
// long enough that the per-item work (q fragments, merge, partial store)
// stays small next to the streaming: at least 128 tokens (one stage of the
// two-page-per-warp path), at most 2048.  Between the two, the multiple of
// 128 nearest to the length that would give about six items per resident
// CTA if every sequence had the maximum length: enough items that the
// longest-first tail is short.  Never more than kMaxPartitions partitions.
// Batches too small to fill the GPU even at 128 tokens get one partition per
// CTA of a thread-block cluster instead (cluster mode, see the decode).
int32_t auto_partition(int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t MB,
                       int32_t kv_dtype) {
    const int64_t maxlen = MB * kPageRows;
    const int64_t G = Hq / std::max<int64_t>(1, Hkv);
    const int64_t resident =
        (int64_t)device_sm_count() * decode_ctas_per_sm(D, G, kv_dtype, false, B);
    // Small batches, where even 128-token partitions would not fill one wave
    // of CTAs: split each (sequence, kv head) into up to kMaxClusterCtas
    // partitions, one CTA each, merged inside their thread-block cluster.
    const int64_t pairs = std::max<int64_t>(1, B * Hkv);
    if (pairs * ceil_div(maxlen, 128) <= resident && maxlen > 128) {
        // the largest cluster size of which `pairs` clusters fit at once
        int64_t np = std::min<int64_t>(kMaxClusterCtas, ceil_div(maxlen, kPageRows));
        while (np >= 2 && decode_cluster_capacity((int)np) < pairs) --np;
        if (np >= 2) {
            int64_t Pc = ceil_div(ceil_div(maxlen, np), kPageRows) * kPageRows;
            const int64_t floor_np =
                ceil_div(ceil_div(maxlen, kMaxPartitions), kPageRows) * kPageRows;
            return (int32_t)std::max(Pc, floor_np);
        }
    }
    // About six items per resident CTA if every context had the maximum
    // length.  Few (sequence, kv head) pairs whose contexts are all long gain
    // from long partitions (each item costs its prologue and merge: the 16 x
    // 131k-token batch runs 2 % faster at P = 8192 than at 2048, its 8-bit
    // cache 6 %); many pairs, as in continuous batching, have mostly short
    // contexts below the maximum, where partitions past 2048 tokens leave the
    // long ones to finish alone (the 256-sequence mix: 1 % slower at 4096).
    const int64_t target_items = 6 * resident;
    const int64_t cap = pairs <= 256 ? PKV_MAX_PARTITION_TOKENS : 2048;
    int64_t P = ceil_div(std::max<int64_t>(1, maxlen * B * Hkv), target_items);
    P = (P + 64) / 128 * 128;
    P = std::max<int64_t>(128, std::min<int64_t>(P, cap));
    const int64_t floor_np = ceil_div(ceil_div(maxlen, kMaxPartitions), kStageTokens) * kStageTokens;
    P = std::max(P, floor_np);
    return (int32_t)P;
}

// Workspace: [scheduler counters, kSchedBytes][partial outputs][partial (m, l)].
// The counters must be zero before the first launch; every launch leaves them zero.
constexpr size_t kSchedBytes = 256;

struct WorkspacePlan {
    int32_t P;
    int32_t NP;
    size_t off_o;
    size_t off_ml;
    size_t bytes;
};

pkv_status plan_workspace(int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t MB,
                          int32_t kv_dtype, int32_t partition_tokens, WorkspacePlan* out) {
    int32_t P = partition_tokens;
    if (P == 0) {
        P = auto_partition(B, Hq, Hkv, D, MB, kv_dtype);
    } else if (P < kPageRows || P % kPageRows != 0 || P > PKV_MAX_PARTITION_TOKENS) {
        set_last_error("partition_tokens %d must be a multiple of 16 in [16, %d]", P,
                       PKV_MAX_PARTITION_TOKENS);
        return PKV_ERR_INVALID_ARG;
    }
    const int64_t NP = std::max<int64_t>(1, ceil_div(MB * kPageRows, P));
    if (NP > kMaxPartitions) {
        set_last_error("max_blocks_per_seq*16 / partition_tokens = %lld partitions > %d",
                       (long long)NP, kMaxPartitions);
        return PKV_ERR_UNSUPPORTED;
    }
    out->P = P;
    out->NP = (int32_t)NP;
    out->off_o = kSchedBytes;
    if (NP <= 1) {
        out->off_ml = kSchedBytes;
        out->bytes = kSchedBytes;
        return PKV_OK;
    }
    const size_t slots = (size_t)B * Hq * NP;
    out->off_ml = out->off_o + align_up(slots * D * sizeof(float));
    out->bytes = out->off_ml + align_up(slots * 2 * sizeof(float));
    return PKV_OK;
}

// Partition length of a sliding-window call that left the choice to the
// library.  The planned length (pkv_decode_workspace_size knows no window)
// suits whole contexts, but a query reads at most window + 15 tokens from
// its window's page on.  Where the planned length would then leave fewer
// work items than resident CTAs, a length chosen for that span gives more,
// as long as its partitions still fit the planned partial slots (the 16 x
// 131k batch at W = 8192: 99 us instead of 163 us at the planned 8192).
int32_t window_partition(int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t MB,
                         int32_t kv_dtype, int32_t window, int32_t P0, int32_t NP0) {
    if (window <= 0) return P0;
    const int64_t span = std::min<int64_t>(MB * kPageRows, (int64_t)window + kPageRows);
    const int64_t G = Hq / std::max<int64_t>(1, Hkv);
    const int64_t resident =
        (int64_t)device_sm_count() * decode_ctas_per_sm(D, G, kv_dtype, false, B);
    if (B * Hkv * ceil_div(span, P0) >= resident) return P0;
    const int64_t mb_w = ceil_div(span, kPageRows);
    const int32_t Pw = auto_partition(B, Hq, Hkv, D, mb_w, kv_dtype);
    if (Pw < P0 && ceil_div(span, Pw) <= NP0) return Pw;
    return P0;
}

pkv_status cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return PKV_OK;
    set_last_error("%s: %s", what, cudaGetErrorString(e));
    return PKV_ERR_CUDA;
}
}  // namespace

}  // namespace pkv

using namespace pkv;

namespace {
// Validation and launch shared by pkv_kv_append and pkv_kv_append_e4m3
// (e4m3: the caches are 8-bit, the scales apply).
pkv_status append_common(void* q, const void* k_new, const void* v_new, const int64_t* positions,
                         const int64_t* slot_mapping, void* k_cache, void* v_cache,
                         int64_t num_tokens, int64_t num_q_heads, int64_t num_kv_heads,
                         int64_t head_dim, int64_t num_blocks, int64_t block_size, int32_t dtype,
                         double rope_theta, int32_t* device_error, void* stream, bool e4m3,
                         float k_scale, float v_scale) {
    if (num_tokens < 0) {
        set_last_error("num_tokens < 0");
        return PKV_ERR_INVALID_ARG;
    }
    pkv_status st = check_heads(num_q_heads, num_kv_heads, head_dim, block_size);
    if (st != PKV_OK) return st;
    if (!valid_dtype(dtype)) {
        set_last_error("dtype %d unsupported", dtype);
        return PKV_ERR_UNSUPPORTED;
    }
    if (!(rope_theta > 0.0)) {
        set_last_error("rope_theta must be > 0");
        return PKV_ERR_INVALID_ARG;
    }
    if (num_blocks <= 0 || num_blocks * num_kv_heads * kPageRows > INT32_MAX) {
        set_last_error("num_blocks %lld out of range", (long long)num_blocks);
        return PKV_ERR_INVALID_ARG;
    }
    if (num_tokens > INT32_MAX) {
        set_last_error("num_tokens too large");
        return PKV_ERR_UNSUPPORTED;
    }
    if (num_tokens == 0) return PKV_OK;
    if (!q || !k_new || !v_new || !positions || !slot_mapping || !k_cache || !v_cache) {
        set_last_error("null tensor pointer");
        return PKV_ERR_INVALID_ARG;
    }
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
        !aligned16(v_cache) || !aligned8(positions) || !aligned8(slot_mapping) ||
        (device_error && !aligned4(device_error))) {
        set_last_error("misaligned tensor pointer (16 bytes for q/k/v/caches)");
        return PKV_ERR_INVALID_ARG;
    }
    AppendArgs a = {};
    a.q = q;
    a.k_new = k_new;
    a.v_new = v_new;
    a.positions = positions;
    a.slot_mapping = slot_mapping;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.num_tokens = num_tokens;
    a.Hq = num_q_heads;
    a.Hkv = num_kv_heads;
    a.D = head_dim;
    a.num_blocks = num_blocks;
    a.dtype = dtype;
    a.theta = rope_theta;
    a.device_error = device_error;
    a.stream = static_cast<cudaStream_t>(stream);
    a.e4m3 = e4m3;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    return cuda_status(launch_kv_append(a), "kv_append launch");
}
}  // namespace

extern "C" {

pkv_status pkv_kv_append(void* q, const void* k_new, const void* v_new, const int64_t* positions,
                         const int64_t* slot_mapping, void* k_cache, void* v_cache,
                         int64_t num_tokens, int64_t num_q_heads, int64_t num_kv_heads,
                         int64_t head_dim, int64_t num_blocks, int64_t block_size, int32_t dtype,
                         double rope_theta, int32_t* device_error, void* stream) {
    set_last_error("");
    return append_common(q, k_new, v_new, positions, slot_mapping, k_cache, v_cache, num_tokens,
                         num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, dtype,
                         rope_theta, device_error, stream, false, 1.f, 1.f);
}

int32_t pkv_decode_partition_tokens(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                    int64_t head_dim, int64_t max_blocks_per_seq,
                                    int64_t block_size, int32_t kv_dtype) {
    if (num_seqs < 0 || max_blocks_per_seq < 0 || !valid_kv_dtype(kv_dtype)) return 0;
    if (check_heads(num_q_heads, num_kv_heads, head_dim, block_size) != PKV_OK) return 0;
    WorkspacePlan w;
    if (plan_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, kv_dtype,
                       0, &w) != PKV_OK)
        return 0;
    return w.P;
}

size_t pkv_decode_workspace_size(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                 int64_t head_dim, int64_t max_blocks_per_seq, int64_t block_size,
                                 int32_t kv_dtype, int32_t partition_tokens) {
    if (num_seqs < 0 || max_blocks_per_seq < 0 || !valid_kv_dtype(kv_dtype)) return 0;
    if (check_heads(num_q_heads, num_kv_heads, head_dim, block_size) != PKV_OK) return 0;
    WorkspacePlan w;
    if (plan_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, kv_dtype,
                       partition_tokens, &w) != PKV_OK)
        return 0;
    return w.bytes;
}

int32_t pkv_decode_launches(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                            int64_t head_dim, int64_t max_blocks_per_seq, int64_t block_size,
                            int32_t kv_dtype, int32_t out_dtype, int32_t partition_tokens,
                            uint32_t flags, int32_t fused) {
    if (num_seqs <= 0 || max_blocks_per_seq <= 0 || !valid_kv_dtype(kv_dtype) ||
        !valid_dtype(out_dtype) || (flags & ~(PKV_DECODE_FORCE_SIMT | PKV_DECODE_NO_CLUSTER)))
        return 0;
    if (kv_dtype == PKV_DTYPE_E4M3 && (flags & PKV_DECODE_FORCE_SIMT)) return 0;
    if (num_seqs > PKV_MAX_SEQS_PER_CALL) return 0;
    if (check_heads(num_q_heads, num_kv_heads, head_dim, block_size) != PKV_OK) return 0;
    WorkspacePlan w;
    if (plan_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, kv_dtype,
                       partition_tokens, &w) != PKV_OK)
        return 0;
    DecodeArgs a = {};
    a.B = num_seqs;
    a.Hq = num_q_heads;
    a.Hkv = num_kv_heads;
    a.D = head_dim;
    a.num_blocks = 1;
    a.MB = max_blocks_per_seq;
    a.kv_dtype = kv_dtype;
    a.out_dtype = out_dtype;
    a.partition_tokens = w.P;
    a.max_partitions = w.NP;
    a.force_simt = (flags & PKV_DECODE_FORCE_SIMT) != 0;
    a.allow_cluster = (flags & PKV_DECODE_NO_CLUSTER) == 0;
    a.fused = fused != 0;
    a.plan_only = true;
    int32_t n = 0;
    a.launches = &n;
    if (launch_paged_decode(a) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    return n;
}

}  // extern "C"

namespace {

struct StepExtras {
    const void* k_new;
    const void* v_new;
    const int64_t* positions;
    const int64_t* slot_mapping;
    double theta;
};

// Shared by the decode call and the fused step: validate, plan, launch.
pkv_status decode_common(const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, const int32_t* context_lens, void* out,
                         void* workspace, size_t workspace_bytes, int64_t num_seqs,
                         int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                         int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq,
                         int32_t kv_dtype, int32_t out_dtype, float scale,
                         int32_t partition_tokens, uint32_t flags, int32_t* device_error,
                         void* stream, const StepExtras* step, const float* kv_scales = nullptr,
                         int32_t window = 0) {
    if (num_seqs < 0 || max_blocks_per_seq < 0) {
        set_last_error("negative num_seqs or max_blocks_per_seq");
        return PKV_ERR_INVALID_ARG;
    }
    pkv_status st = check_heads(num_q_heads, num_kv_heads, head_dim, block_size);
    if (st != PKV_OK) return st;
    if (kv_dtype == PKV_DTYPE_E4M3 && !kv_scales) {
        set_last_error("the 8-bit cache is decoded by pkv_paged_attention_decode_e4m3");
        return PKV_ERR_UNSUPPORTED;
    }
    if (!valid_kv_dtype(kv_dtype) || !valid_dtype(out_dtype)) {
        set_last_error("kv_dtype/out_dtype unsupported");
        return PKV_ERR_UNSUPPORTED;
    }
    if (kv_dtype == PKV_DTYPE_E4M3) {
        if (flags & PKV_DECODE_FORCE_SIMT) {
            set_last_error("the 8-bit cache has no CUDA-core kernel");
            return PKV_ERR_UNSUPPORTED;
        }
        for (int i = 0; i < 2; ++i)
            if (!(kv_scales[i] > 0.f) || kv_scales[i] == INFINITY) {
                set_last_error("k_scale and v_scale must be finite and > 0");
                return PKV_ERR_INVALID_ARG;
            }
        if (num_blocks * num_kv_heads * head_dim > INT32_MAX) {
            set_last_error("num_blocks %lld too large for the 8-bit cache", (long long)num_blocks);
            return PKV_ERR_INVALID_ARG;
        }
    }
    if ((flags & ~(PKV_DECODE_FORCE_SIMT | PKV_DECODE_NO_CLUSTER)) != 0) {
        set_last_error("unknown flags 0x%x", flags);
        return PKV_ERR_INVALID_ARG;
    }
    if (num_seqs > PKV_MAX_SEQS_PER_CALL) {
        set_last_error("num_seqs %lld > %d", (long long)num_seqs, PKV_MAX_SEQS_PER_CALL);
        return PKV_ERR_UNSUPPORTED;
    }
    if (num_blocks <= 0 || num_blocks * num_kv_heads * kPageRows > INT32_MAX) {
        set_last_error("num_blocks %lld out of range", (long long)num_blocks);
        return PKV_ERR_INVALID_ARG;
    }
    if (max_blocks_per_seq * kPageRows > INT32_MAX / 2) {
        set_last_error("max_blocks_per_seq too large");
        return PKV_ERR_UNSUPPORTED;
    }
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY) {
        set_last_error("scale must be finite");
        return PKV_ERR_INVALID_ARG;
    }
    if (step && !(step->theta > 0.0)) {
        set_last_error("rope_theta must be > 0");
        return PKV_ERR_INVALID_ARG;
    }
    if (window < 0) {
        set_last_error("sliding_window must be >= 0");
        return PKV_ERR_INVALID_ARG;
    }
    WorkspacePlan w;
    st = plan_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                        kv_dtype, partition_tokens, &w);
    if (st != PKV_OK) return st;
    if (num_seqs == 0) return PKV_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) {
        set_last_error("null tensor pointer");
        return PKV_ERR_INVALID_ARG;
    }
    if (step && (!step->k_new || !step->v_new || !step->positions || !step->slot_mapping)) {
        set_last_error("null tensor pointer");
        return PKV_ERR_INVALID_ARG;
    }
    if (max_blocks_per_seq == 0) {
        set_last_error("max_blocks_per_seq must be > 0 when num_seqs > 0");
        return PKV_ERR_INVALID_ARG;
    }
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        !aligned4(block_tables) || !aligned4(context_lens) ||
        (device_error && !aligned4(device_error)) ||
        (step && (!aligned16(step->k_new) || !aligned16(step->v_new) ||
                  !aligned8(step->positions) || !aligned8(step->slot_mapping)))) {
        set_last_error("misaligned tensor pointer (16 bytes for q/k/v/caches/out)");
        return PKV_ERR_INVALID_ARG;
    }
    // With one partition per sequence the workspace is optional: without it
    // the work items are dealt out statically instead of claimed.
    const bool have_ws = workspace && workspace_bytes >= w.bytes;
    if ((w.NP > 1 && !have_ws) || (have_ws && !aligned16(workspace))) {
        set_last_error("workspace of %zu bytes given, %zu needed (16-byte aligned)",
                       workspace ? workspace_bytes : (size_t)0, w.bytes);
        return PKV_ERR_WORKSPACE;
    }
    DecodeArgs a = {};
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.out = out;
    char* ws = static_cast<char*>(workspace);
    a.sched = have_ws ? reinterpret_cast<uint32_t*>(ws) : nullptr;
    a.part_o = (have_ws && w.NP > 1) ? reinterpret_cast<float*>(ws + w.off_o) : nullptr;
    a.part_ml = (have_ws && w.NP > 1) ? reinterpret_cast<float*>(ws + w.off_ml) : nullptr;
    a.B = num_seqs;
    a.Hq = num_q_heads;
    a.Hkv = num_kv_heads;
    a.D = head_dim;
    a.num_blocks = num_blocks;
    a.MB = max_blocks_per_seq;
    a.kv_dtype = kv_dtype;
    a.out_dtype = out_dtype;
    a.k_scale = kv_scales ? kv_scales[0] : 1.f;
    a.v_scale = kv_scales ? kv_scales[1] : 1.f;
    a.partition_tokens = partition_tokens == 0
                             ? window_partition(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                max_blocks_per_seq, kv_dtype, window, w.P, w.NP)
                             : w.P;
    a.max_partitions = w.NP;  // the partial slots per row the workspace holds
    a.scale = scale;
    a.force_simt = (flags & PKV_DECODE_FORCE_SIMT) != 0;
    a.allow_cluster = (flags & PKV_DECODE_NO_CLUSTER) == 0;
    a.device_error = device_error;
    a.stream = static_cast<cudaStream_t>(stream);
    a.window = window;
    a.fused = step != nullptr;
    if (step) {
        a.k_new = step->k_new;
        a.v_new = step->v_new;
        a.positions = step->positions;
        a.slot_mapping = step->slot_mapping;
        a.theta = step->theta;
    }
    return cuda_status(launch_paged_decode(a), step ? "decode_step launch"
                                                    : "paged_attention_decode launch");
}

}  // namespace

extern "C" {

pkv_status pkv_paged_attention_decode(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, const int32_t* context_lens,
                                      void* out, void* workspace, size_t workspace_bytes,
                                      int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                      int64_t head_dim, int64_t num_blocks, int64_t block_size,
                                      int64_t max_blocks_per_seq, int32_t kv_dtype,
                                      int32_t out_dtype, float scale, int32_t partition_tokens,
                                      uint32_t flags, int32_t* device_error, void* stream) {
    set_last_error("");
    return decode_common(q, k_cache, v_cache, block_tables, context_lens, out, workspace,
                         workspace_bytes, num_seqs, num_q_heads, num_kv_heads, head_dim,
                         num_blocks, block_size, max_blocks_per_seq, kv_dtype, out_dtype, scale,
                         partition_tokens, flags, device_error, stream, nullptr);
}

pkv_status pkv_decode_step(void* q, const void* k_new, const void* v_new, const int64_t* positions,
                           const int64_t* slot_mapping, void* k_cache, void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens, void* out,
                           void* workspace, size_t workspace_bytes, int64_t num_seqs,
                           int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                           int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq,
                           int32_t kv_dtype, int32_t out_dtype, double rope_theta, float scale,
                           int32_t partition_tokens, uint32_t flags, int32_t* device_error,
                           void* stream) {
    set_last_error("");
    const StepExtras step = {k_new, v_new, positions, slot_mapping, rope_theta};
    return decode_common(q, k_cache, v_cache, block_tables, context_lens, out, workspace,
                         workspace_bytes, num_seqs, num_q_heads, num_kv_heads, head_dim,
                         num_blocks, block_size, max_blocks_per_seq, kv_dtype, out_dtype, scale,
                         partition_tokens, flags, device_error, stream, &step);
}

pkv_status pkv_decode_step_window(void* q, const void* k_new, const void* v_new,
                                  const int64_t* positions, const int64_t* slot_mapping,
                                  void* k_cache, void* v_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, void* out, void* workspace,
                                  size_t workspace_bytes, int64_t num_seqs, int64_t num_q_heads,
                                  int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                                  int64_t block_size, int64_t max_blocks_per_seq,
                                  int32_t kv_dtype, int32_t out_dtype, double rope_theta,
                                  float scale, int32_t sliding_window, int32_t partition_tokens,
                                  uint32_t flags, int32_t* device_error, void* stream) {
    set_last_error("");
    const StepExtras step = {k_new, v_new, positions, slot_mapping, rope_theta};
    return decode_common(q, k_cache, v_cache, block_tables, context_lens, out, workspace,
                         workspace_bytes, num_seqs, num_q_heads, num_kv_heads, head_dim,
                         num_blocks, block_size, max_blocks_per_seq, kv_dtype, out_dtype, scale,
                         partition_tokens, flags, device_error, stream, &step, nullptr,
                         sliding_window);
}

pkv_status pkv_paged_attention_decode_e4m3(const void* q, const void* kv_cache,
                                           const int32_t* block_tables,
                                           const int32_t* context_lens, void* out,
                                           void* workspace, size_t workspace_bytes,
                                           int64_t num_seqs, int64_t num_q_heads,
                                           int64_t num_kv_heads, int64_t head_dim,
                                           int64_t num_blocks, int64_t block_size,
                                           int64_t max_blocks_per_seq, int32_t out_dtype,
                                           float scale, float k_scale, float v_scale,
                                           int32_t sliding_window, int32_t partition_tokens,
                                           uint32_t flags, int32_t* device_error, void* stream) {
    set_last_error("");
    const float scales[2] = {k_scale, v_scale};
    // one [K | V] region per page: both halves are reached from kv_cache
    return decode_common(q, kv_cache, kv_cache, block_tables, context_lens, out, workspace,
                         workspace_bytes, num_seqs, num_q_heads, num_kv_heads, head_dim,
                         num_blocks, block_size, max_blocks_per_seq, PKV_DTYPE_E4M3, out_dtype,
                         scale, partition_tokens, flags, device_error, stream, nullptr, scales,
                         sliding_window);
}

pkv_status pkv_decode_step_e4m3(void* q, const void* k_new, const void* v_new,
                                const int64_t* positions, const int64_t* slot_mapping,
                                void* kv_cache, const int32_t* block_tables,
                                const int32_t* context_lens, void* out, void* workspace,
                                size_t workspace_bytes, int64_t num_seqs, int64_t num_q_heads,
                                int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                                int64_t block_size, int64_t max_blocks_per_seq, int32_t out_dtype,
                                double rope_theta, float scale, float k_scale, float v_scale,
                                int32_t sliding_window, int32_t partition_tokens, uint32_t flags,
                                int32_t* device_error, void* stream) {
    set_last_error("");
    const float scales[2] = {k_scale, v_scale};
    const StepExtras step = {k_new, v_new, positions, slot_mapping, rope_theta};
    return decode_common(q, kv_cache, kv_cache, block_tables, context_lens, out, workspace,
                         workspace_bytes, num_seqs, num_q_heads, num_kv_heads, head_dim,
                         num_blocks, block_size, max_blocks_per_seq, PKV_DTYPE_E4M3, out_dtype,
                         scale, partition_tokens, flags, device_error, stream, &step, scales,
                         sliding_window);
}

pkv_status pkv_paged_attention_decode_window(const void* q, const void* k_cache,
                                             const void* v_cache, const int32_t* block_tables,
                                             const int32_t* context_lens, void* out,
                                             void* workspace, size_t workspace_bytes,
                                             int64_t num_seqs, int64_t num_q_heads,
                                             int64_t num_kv_heads, int64_t head_dim,
                                             int64_t num_blocks, int64_t block_size,
                                             int64_t max_blocks_per_seq, int32_t kv_dtype,
                                             int32_t out_dtype, float scale,
                                             int32_t sliding_window, int32_t partition_tokens,
                                             uint32_t flags, int32_t* device_error,
                                             void* stream) {
    set_last_error("");
    return decode_common(q, k_cache, v_cache, block_tables, context_lens, out, workspace,
                         workspace_bytes, num_seqs, num_q_heads, num_kv_heads, head_dim,
                         num_blocks, block_size, max_blocks_per_seq, kv_dtype, out_dtype, scale,
                         partition_tokens, flags, device_error, stream, nullptr, nullptr,
                         sliding_window);
}

pkv_status pkv_kv_append_e4m3(void* q, const void* k_new, const void* v_new,
                              const int64_t* positions, const int64_t* slot_mapping,
                              void* kv_cache, int64_t num_tokens,
                              int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                              int64_t num_blocks, int64_t block_size, int32_t dtype,
                              double rope_theta, float k_scale, float v_scale,
                              int32_t* device_error, void* stream) {
    set_last_error("");
    if (!(k_scale > 0.f) || k_scale == INFINITY || !(v_scale > 0.f) || v_scale == INFINITY) {
        set_last_error("k_scale and v_scale must be finite and > 0");
        return PKV_ERR_INVALID_ARG;
    }
    if (num_blocks > 0 && num_kv_heads > 0 && head_dim > 0 &&
        num_blocks * num_kv_heads * head_dim > INT32_MAX) {
        set_last_error("num_blocks %lld too large for the 8-bit cache", (long long)num_blocks);
        return PKV_ERR_INVALID_ARG;
    }
    return append_common(q, k_new, v_new, positions, slot_mapping, kv_cache, kv_cache,
                         num_tokens, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size,
                         dtype, rope_theta, device_error, stream, true, k_scale, v_scale);
}

}  // extern "C"

// ---- cascade decode ----------------------------------------------------------

namespace pkv {
namespace {
cudaError_t launch_cascade_between(const void* ctx) {
    return launch_cascade_prefix(*static_cast<const CascadeArgs*>(ctx));
}

// Workspace of a cascade call: the scheduler counters, then NP + 1 partial
// slots per (sequence, q head) -- slot 0 for the shared prefix.
pkv_status plan_cascade(int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t MB,
                        int32_t kv_dtype, int32_t partition_tokens, WorkspacePlan* w,
                        int32_t* slots_per_row) {
    pkv_status st = plan_workspace(B, Hq, Hkv, D, MB, kv_dtype, partition_tokens, w);
    if (st != PKV_OK) return st;
    if (w->NP + 1 > kMaxPartitions) {
        set_last_error("cascade: at most %d partitions per sequence", kMaxPartitions - 1);
        return PKV_ERR_UNSUPPORTED;
    }
    *slots_per_row = w->NP + 1;
    const size_t slots = (size_t)B * Hq * (w->NP + 1);
    w->off_o = kSchedBytes;
    w->off_ml = w->off_o + align_up(slots * D * sizeof(float));
    w->bytes = w->off_ml + align_up(slots * 2 * sizeof(float));
    return PKV_OK;
}
}  // namespace
}  // namespace pkv

extern "C" {

size_t pkv_decode_cascade_workspace_size(int64_t num_seqs, int64_t num_q_heads,
                                         int64_t num_kv_heads, int64_t head_dim,
                                         int64_t max_blocks_per_seq, int64_t block_size,
                                         int32_t kv_dtype, int32_t partition_tokens) {
    if (num_seqs < 0 || max_blocks_per_seq < 0 || kv_dtype != PKV_DTYPE_BF16) return 0;
    if (check_heads(num_q_heads, num_kv_heads, head_dim, block_size) != PKV_OK) return 0;
    WorkspacePlan w;
    int32_t npt;
    if (plan_cascade(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, kv_dtype,
                     partition_tokens, &w, &npt) != PKV_OK)
        return 0;
    return w.bytes;
}

}  // extern "C"

namespace {
pkv_status cascade_common(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* context_lens, const int32_t* group_start, const int32_t* shared_tokens,
    void* out, void* workspace, size_t workspace_bytes, int64_t num_seqs, int64_t num_groups,
    int64_t max_group_size, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
    int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq, int32_t kv_dtype,
    int32_t out_dtype, float scale, int32_t window, int32_t partition_tokens, uint32_t flags,
    int32_t* device_error, void* stream) {
    if (num_seqs < 0 || max_blocks_per_seq < 0 || num_groups < 0) {
        set_last_error("negative num_seqs, num_groups or max_blocks_per_seq");
        return PKV_ERR_INVALID_ARG;
    }
    pkv_status st = check_heads(num_q_heads, num_kv_heads, head_dim, block_size);
    if (st != PKV_OK) return st;
    if (kv_dtype != PKV_DTYPE_BF16 || !valid_dtype(out_dtype)) {
        set_last_error("cascade: kv_dtype must be bf16; out_dtype f32 or bf16");
        return PKV_ERR_UNSUPPORTED;
    }
    if ((flags & ~PKV_DECODE_FORCE_SIMT) != 0) {
        set_last_error("cascade: unknown flags 0x%x", flags);
        return PKV_ERR_INVALID_ARG;
    }
    if (num_seqs > kCascadeMaxSeqs) {
        set_last_error("cascade: num_seqs %lld > %d", (long long)num_seqs, kCascadeMaxSeqs);
        return PKV_ERR_UNSUPPORTED;
    }
    if (num_groups > 0 && (max_group_size < 1 || max_group_size > num_seqs ||
                           num_groups * num_kv_heads *
                                   ceil_div(max_group_size * (num_q_heads / num_kv_heads), 32) >
                               INT32_MAX)) {
        set_last_error("cascade: max_group_size %lld out of range", (long long)max_group_size);
        return PKV_ERR_INVALID_ARG;
    }
    if (num_blocks <= 0 || num_blocks * num_kv_heads * kPageRows > INT32_MAX) {
        set_last_error("num_blocks %lld out of range", (long long)num_blocks);
        return PKV_ERR_INVALID_ARG;
    }
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY) {
        set_last_error("scale must be finite");
        return PKV_ERR_INVALID_ARG;
    }
    if (window < 0) {
        set_last_error("sliding_window must be >= 0");
        return PKV_ERR_INVALID_ARG;
    }
    WorkspacePlan w;
    int32_t npt;
    st = plan_cascade(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, kv_dtype,
                      partition_tokens, &w, &npt);
    if (st != PKV_OK) return st;
    if (num_seqs == 0) return PKV_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out || !shared_tokens ||
        (num_groups > 0 && !group_start)) {
        set_last_error("null tensor pointer");
        return PKV_ERR_INVALID_ARG;
    }
    if (max_blocks_per_seq == 0) {
        set_last_error("max_blocks_per_seq must be > 0 when num_seqs > 0");
        return PKV_ERR_INVALID_ARG;
    }
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        !aligned4(block_tables) || !aligned4(context_lens) || !aligned4(shared_tokens) ||
        (group_start && !aligned4(group_start)) || (device_error && !aligned4(device_error))) {
        set_last_error("misaligned tensor pointer");
        return PKV_ERR_INVALID_ARG;
    }
    if (!workspace || workspace_bytes < w.bytes || !aligned16(workspace)) {
        set_last_error("workspace of %zu bytes given, %zu needed (16-byte aligned)",
                       workspace ? workspace_bytes : (size_t)0, w.bytes);
        return PKV_ERR_WORKSPACE;
    }
    char* ws = static_cast<char*>(workspace);
    CascadeArgs c = {};
    c.q = q;
    c.k_cache = k_cache;
    c.v_cache = v_cache;
    c.block_tables = block_tables;
    c.context_lens = context_lens;
    c.group_start = group_start;
    c.shared_tokens = shared_tokens;
    c.part_o = reinterpret_cast<float*>(ws + w.off_o);
    c.part_ml = reinterpret_cast<float*>(ws + w.off_ml);
    c.B = num_seqs;
    c.Hq = num_q_heads;
    c.Hkv = num_kv_heads;
    c.D = head_dim;
    c.num_blocks = num_blocks;
    c.MB = max_blocks_per_seq;
    c.num_groups = num_groups;
    c.max_group_size = max_group_size;
    c.slots_per_row = npt;
    c.window = window;
    c.scale = scale;
    c.device_error = device_error;
    c.stream = static_cast<cudaStream_t>(stream);

    DecodeArgs a = {};
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.out = out;
    a.sched = reinterpret_cast<uint32_t*>(ws);
    a.part_o = c.part_o;
    a.part_ml = c.part_ml;
    a.B = num_seqs;
    a.Hq = num_q_heads;
    a.Hkv = num_kv_heads;
    a.D = head_dim;
    a.num_blocks = num_blocks;
    a.MB = max_blocks_per_seq;
    a.kv_dtype = kv_dtype;
    a.out_dtype = out_dtype;
    a.partition_tokens = partition_tokens == 0
                             ? window_partition(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                max_blocks_per_seq, kv_dtype, window, w.P, w.NP)
                             : w.P;
    a.max_partitions = npt;   // the slot stride: the shared slot, then the partitions
    a.scale = scale;
    a.force_simt = (flags & PKV_DECODE_FORCE_SIMT) != 0;
    a.allow_cluster = false;
    a.shared_tokens = shared_tokens;
    a.window = window;
    a.launch_between = launch_cascade_between;
    a.between_ctx = &c;
    a.device_error = device_error;
    a.stream = static_cast<cudaStream_t>(stream);
    return cuda_status(launch_paged_decode(a), "cascade decode launch");
}
}  // namespace

extern "C" {

pkv_status pkv_paged_attention_decode_cascade(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* context_lens, const int32_t* group_start, const int32_t* shared_tokens,
    void* out, void* workspace, size_t workspace_bytes, int64_t num_seqs, int64_t num_groups,
    int64_t max_group_size, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
    int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq, int32_t kv_dtype,
    int32_t out_dtype, float scale, int32_t partition_tokens, uint32_t flags,
    int32_t* device_error, void* stream) {
    set_last_error("");
    return cascade_common(q, k_cache, v_cache, block_tables, context_lens, group_start,
                          shared_tokens, out, workspace, workspace_bytes, num_seqs, num_groups,
                          max_group_size, num_q_heads, num_kv_heads, head_dim, num_blocks,
                          block_size, max_blocks_per_seq, kv_dtype, out_dtype, scale, 0,
                          partition_tokens, flags, device_error, stream);
}

pkv_status pkv_paged_attention_decode_cascade_window(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* context_lens, const int32_t* group_start, const int32_t* shared_tokens,
    void* out, void* workspace, size_t workspace_bytes, int64_t num_seqs, int64_t num_groups,
    int64_t max_group_size, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
    int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq, int32_t kv_dtype,
    int32_t out_dtype, float scale, int32_t sliding_window, int32_t partition_tokens,
    uint32_t flags, int32_t* device_error, void* stream) {
    set_last_error("");
    return cascade_common(q, k_cache, v_cache, block_tables, context_lens, group_start,
                          shared_tokens, out, workspace, workspace_bytes, num_seqs, num_groups,
                          max_group_size, num_q_heads, num_kv_heads, head_dim, num_blocks,
                          block_size, max_blocks_per_seq, kv_dtype, out_dtype, scale,
                          sliding_window, partition_tokens, flags, device_error, stream);
}

}  // extern "C"

// ---- chunked prefill ---------------------------------------------------------

namespace pkv {
namespace {
constexpr int kPrefillRowsPerItem = 128;  // (query, head) rows one prefill CTA serves

// Partition length of a prefill call: about two items per SM (one CTA per SM
// at a time) if every sequence had the maximum length, in whole 64-key tiles,
// [256, PKV_MAX_PARTITION_TOKENS].  An item pays about 6 us of set-up,
// pipeline fill and epilogue, so few long items beat many short ones (on the
// ragged batch at C = 16: 144 us at P = 4096 against 167 us at P = 1792, the
// earlier choice of eight items per SM); only where the items are then fewer
// than the SMs do shorter partitions win (batch 1, 2048 tokens: P = 256).
int32_t prefill_auto_partition(int64_t B, int64_t C, int64_t Hq, int64_t Hkv, int64_t MB) {
    const int64_t maxlen = MB * kPageRows;
    const int64_t G = Hq / std::max<int64_t>(1, Hkv);
    const int64_t rg = ceil_div(C * G, kPrefillRowsPerItem);
    const int64_t target = 2 * (int64_t)device_sm_count();
    int64_t P = ceil_div(std::max<int64_t>(1, maxlen * B * Hkv * rg), target);
    P = ceil_div(P, 64) * 64;
    P = std::max<int64_t>(256, std::min<int64_t>(P, PKV_MAX_PARTITION_TOKENS));
    const int64_t floor_np = ceil_div(ceil_div(maxlen, kMaxPartitions), kPageRows) * kPageRows;
    return (int32_t)std::max(P, floor_np);
}

pkv_status plan_prefill(int64_t B, int64_t C, int64_t Hq, int64_t Hkv, int64_t D, int64_t MB,
                        int32_t partition_tokens, int32_t* P_out, int32_t* NP_out,
                        size_t* off_ml, size_t* bytes) {
    int32_t P = partition_tokens;
    if (P == 0) {
        P = prefill_auto_partition(B, C, Hq, Hkv, MB);
    } else if (P < kPageRows || P % kPageRows != 0 || P > PKV_MAX_PARTITION_TOKENS) {
        set_last_error("partition_tokens %d must be a multiple of 16 in [16, %d]", P,
                       PKV_MAX_PARTITION_TOKENS);
        return PKV_ERR_INVALID_ARG;
    }
    const int64_t NP = std::max<int64_t>(1, ceil_div(MB * kPageRows, P));
    if (NP > kMaxPartitions) {
        set_last_error("max_blocks_per_seq*16 / partition_tokens = %lld partitions > %d",
                       (long long)NP, kMaxPartitions);
        return PKV_ERR_UNSUPPORTED;
    }
    *P_out = P;
    *NP_out = (int32_t)NP;
    const size_t slots = NP > 1 ? (size_t)B * C * Hq * NP : 0;
    *off_ml = align_up(slots * D * sizeof(float));
    *bytes = slots ? *off_ml + align_up(slots * 2 * sizeof(float)) : 0;
    return PKV_OK;
}
}  // namespace
}  // namespace pkv

extern "C" {

int32_t pkv_prefill_partition_tokens(int64_t num_seqs, int64_t chunk_tokens, int64_t num_q_heads,
                                     int64_t num_kv_heads, int64_t head_dim,
                                     int64_t max_blocks_per_seq, int64_t block_size) {
    if (num_seqs < 0 || chunk_tokens < 1 || max_blocks_per_seq < 0) return 0;
    if (check_heads(num_q_heads, num_kv_heads, head_dim, block_size) != PKV_OK) return 0;
    return prefill_auto_partition(num_seqs, chunk_tokens, num_q_heads, num_kv_heads,
                                  max_blocks_per_seq);
}

size_t pkv_prefill_workspace_size(int64_t num_seqs, int64_t chunk_tokens, int64_t num_q_heads,
                                  int64_t num_kv_heads, int64_t head_dim,
                                  int64_t max_blocks_per_seq, int64_t block_size,
                                  int32_t partition_tokens) {
    if (num_seqs < 0 || chunk_tokens < 1 || max_blocks_per_seq < 0) return 0;
    if (check_heads(num_q_heads, num_kv_heads, head_dim, block_size) != PKV_OK) return 0;
    int32_t P, NP;
    size_t off_ml, bytes;
    if (plan_prefill(num_seqs, chunk_tokens, num_q_heads, num_kv_heads, head_dim,
                     max_blocks_per_seq, partition_tokens, &P, &NP, &off_ml, &bytes) != PKV_OK)
        return 0;
    return bytes;
}

pkv_status pkv_paged_attention_prefill(const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       void* out, void* workspace, size_t workspace_bytes,
                                       int64_t num_seqs, int64_t chunk_tokens,
                                       int64_t num_q_heads, int64_t num_kv_heads,
                                       int64_t head_dim, int64_t num_blocks, int64_t block_size,
                                       int64_t max_blocks_per_seq, int32_t kv_dtype,
                                       int32_t out_dtype, float scale, int32_t sliding_window,
                                       int32_t partition_tokens, int32_t* device_error,
                                       void* stream) {
    set_last_error("");
    if (sliding_window < 0) {
        set_last_error("sliding_window must be >= 0");
        return PKV_ERR_INVALID_ARG;
    }
    if (num_seqs < 0 || max_blocks_per_seq < 0 || chunk_tokens < 1) {
        set_last_error("negative num_seqs or max_blocks_per_seq, or chunk_tokens < 1");
        return PKV_ERR_INVALID_ARG;
    }
    pkv_status st = check_heads(num_q_heads, num_kv_heads, head_dim, block_size);
    if (st != PKV_OK) return st;
    if (kv_dtype != PKV_DTYPE_BF16 || !valid_dtype(out_dtype)) {
        set_last_error("prefill: kv_dtype must be bf16; out_dtype f32 or bf16");
        return PKV_ERR_UNSUPPORTED;
    }
    if (num_seqs > PKV_MAX_SEQS_PER_CALL) {
        set_last_error("num_seqs %lld > %d", (long long)num_seqs, PKV_MAX_SEQS_PER_CALL);
        return PKV_ERR_UNSUPPORTED;
    }
    if (chunk_tokens > max_blocks_per_seq * kPageRows && num_seqs > 0) {
        set_last_error("chunk_tokens %lld longer than max_blocks_per_seq * 16",
                       (long long)chunk_tokens);
        return PKV_ERR_INVALID_ARG;
    }
    if (num_blocks <= 0 || num_blocks * num_kv_heads * kPageRows > INT32_MAX) {
        set_last_error("num_blocks %lld out of range", (long long)num_blocks);
        return PKV_ERR_INVALID_ARG;
    }
    if (max_blocks_per_seq * kPageRows > INT32_MAX / 2) {
        set_last_error("max_blocks_per_seq too large");
        return PKV_ERR_UNSUPPORTED;
    }
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY) {
        set_last_error("scale must be finite");
        return PKV_ERR_INVALID_ARG;
    }
    int32_t P, NP;
    size_t off_ml, need;
    st = plan_prefill(num_seqs, chunk_tokens, num_q_heads, num_kv_heads, head_dim,
                      max_blocks_per_seq, partition_tokens, &P, &NP, &off_ml, &need);
    if (st != PKV_OK) return st;
    const int64_t grid = num_seqs * num_kv_heads * NP *
                         ceil_div(chunk_tokens * (num_q_heads / num_kv_heads), kPrefillRowsPerItem);
    if (grid > INT32_MAX) {
        set_last_error("prefill: too many work items");
        return PKV_ERR_UNSUPPORTED;
    }
    if (num_seqs == 0) return PKV_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) {
        set_last_error("null tensor pointer");
        return PKV_ERR_INVALID_ARG;
    }
    if (max_blocks_per_seq == 0) {
        set_last_error("max_blocks_per_seq must be > 0 when num_seqs > 0");
        return PKV_ERR_INVALID_ARG;
    }
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        !aligned4(block_tables) || !aligned4(context_lens) ||
        (device_error && !aligned4(device_error))) {
        set_last_error("misaligned tensor pointer (16 bytes for q/caches/out)");
        return PKV_ERR_INVALID_ARG;
    }
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) {
        set_last_error("workspace of %zu bytes given, %zu needed (16-byte aligned)",
                       workspace ? workspace_bytes : (size_t)0, need);
        return PKV_ERR_WORKSPACE;
    }
    PrefillArgs a = {};
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.out = out;
    a.part_o = need ? static_cast<float*>(workspace) : nullptr;
    a.part_ml = need ? reinterpret_cast<float*>(static_cast<char*>(workspace) + off_ml) : nullptr;
    a.B = num_seqs;
    a.C = chunk_tokens;
    a.Hq = num_q_heads;
    a.Hkv = num_kv_heads;
    a.D = head_dim;
    a.num_blocks = num_blocks;
    a.MB = max_blocks_per_seq;
    a.out_dtype = out_dtype;
    a.partition_tokens = P;
    a.max_partitions = NP;
    a.scale = scale;
    a.window = sliding_window;
    a.device_error = device_error;
    a.stream = static_cast<cudaStream_t>(stream);
    return cuda_status(launch_paged_prefill(a), "prefill launch");
}

const char* pkv_status_string(int32_t status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID_ARG: return "invalid argument";
        case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
        case PKV_ERR_WORKSPACE: return "workspace too small";
        case PKV_ERR_CUDA: return "CUDA error";
        case PKV_ERR_DEVICE: return "device error word set by a kernel";
    }
    return "unknown status";
}

const char* pkv_last_error(void) { return g_last_error; }

int32_t pkv_version(void) { return 200; }

}  // extern "C"
