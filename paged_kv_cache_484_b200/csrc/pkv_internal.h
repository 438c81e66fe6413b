// pkv_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pkv.h"

namespace pkv {

constexpr int kPageRows = 16;      // tokens per cache block (block_size)
constexpr int kConsumerWarps = 4;  // decode: warps that compute
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kStageTokens = kConsumerWarps * kPageRows;   // one page per consumer warp
constexpr int kMaxPartitions = 1024;
constexpr int kMaxClusterCtas = 16;  // cluster-mode limit (non-portable above 8)
constexpr int kCascadeMaxSeqs = 256;  // cascade decode keeps per-sequence offsets in shared memory

// Per-thread detail of the last failing call (returned by pkv_last_error).
void set_last_error(const char* fmt, ...);

struct AppendArgs {
    void* q;
    const void* k_new;
    const void* v_new;
    const int64_t* positions;
    const int64_t* slot_mapping;
    void* k_cache;
    void* v_cache;
    int64_t num_tokens, Hq, Hkv, D, num_blocks;
    int32_t dtype;       // of q, k_new, v_new (and of the caches unless e4m3)
    double theta;
    int32_t* device_error;
    cudaStream_t stream;
    // 8-bit cache: codes of k / k_scale and v / v_scale; V pages transposed
    bool e4m3;
    float k_scale, v_scale;
};
cudaError_t launch_kv_append(const AppendArgs& a);

struct DecodeArgs {
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    void* out;
    float* part_o;   // [B, Hq, NP, D]
    float* part_ml;  // [B, Hq, NP, 2]
    uint32_t* sched; // scheduler counters (2 x u32, zero between launches); null: static
    int64_t B, Hq, Hkv, D, num_blocks, MB;
    int32_t kv_dtype, out_dtype;  // kv_dtype PKV_DTYPE_E4M3: q is bf16
    float k_scale, v_scale;       // 8-bit cache only (1 otherwise)
    int32_t partition_tokens;  // P (resolved, multiple of 16)
    int32_t max_partitions;    // NP = ceil(MB * 16 / P)
    float scale;
    bool force_simt;
    bool allow_cluster;  // split contexts may merge inside a thread-block cluster
    // cascade: tokens of each sequence attended by the shared-prefix pass
    // (partial slot 0), and that pass's launch, made between the decode
    // kernel and the combine; null = no cascade
    const int32_t* shared_tokens;
    int32_t window;  // sliding window, 0 = none (not with shared_tokens)
    cudaError_t (*launch_between)(const void* ctx);
    const void* between_ctx;
    // planning only: launch nothing, store the number of kernels the call
    // would launch (1 or 2) in *launches
    bool plan_only;
    int32_t* launches;
    int32_t* device_error;
    cudaStream_t stream;
    // fused step (append inside the decode kernel); q is rotated in place
    bool fused;
    const void* k_new;
    const void* v_new;
    const int64_t* positions;
    const int64_t* slot_mapping;
    double theta;
};
cudaError_t launch_paged_decode(const DecodeArgs& a);

// The cache [num_blocks, Hkv, 16, D] as a TMA tensor map of 16-row page boxes.
cudaError_t encode_cache_map(CUtensorMap* map, const void* cache, int64_t num_blocks, int64_t Hkv,
                             int64_t D, int32_t dtype);

struct PrefillArgs {
    const void* q;              // [B, C, Hq, D] bf16
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    void* out;                  // [B, C, Hq, D]
    float* part_o;              // [B, C, Hq, NP, D]
    float* part_ml;             // [B, C, Hq, NP, 2]
    int64_t B, C, Hq, Hkv, D, num_blocks, MB;
    int32_t out_dtype;
    int32_t partition_tokens;   // P (resolved)
    int32_t max_partitions;     // NP = ceil(MB * 16 / P)
    float scale;
    int32_t window;             // sliding window, 0 = none
    int32_t* device_error;
    cudaStream_t stream;
};
cudaError_t launch_paged_prefill(const PrefillArgs& a);

// Cascade decode, shared-prefix pass (launched between the decode kernel and
// the combine).
struct CascadeArgs {
    const void* q;                  // [B, Hq, D] bf16, rotated
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* group_start;     // [num_groups + 1]
    const int32_t* shared_tokens;   // [B]
    float* part_o;
    float* part_ml;
    int64_t B, Hq, Hkv, D, num_blocks, MB, num_groups, max_group_size;
    int32_t slots_per_row;          // partial slots per (sequence, q head): 1 + NP
    int32_t window;                 // sliding window (0: none)
    float scale;
    int32_t* device_error;
    cudaStream_t stream;
};
cudaError_t launch_cascade_prefix(const CascadeArgs& a);

// Resident decode CTAs per SM for these shapes (occupancy query, cached).
int decode_ctas_per_sm(int64_t D, int64_t G, int32_t kv_dtype, bool simt, int64_t num_seqs);
int device_sm_count();
// Clusters of `cs` decode CTAs (cluster mode, one CTA per SM) that can be
// resident at once on the current device; 0 when unknown.
int decode_cluster_capacity(int cs);

}  // namespace pkv
