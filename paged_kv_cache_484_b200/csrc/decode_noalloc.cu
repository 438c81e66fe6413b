// decode_noalloc.cu -- paged_attention_decode for callers that cannot allocate.
//
// Some callers of this library cannot hand it a workspace.  Typical cases: a
// serving engine that reserved nearly all device memory for its KV block
// pool at start-up and may not allocate on the decode path; a plugin
// interface that passes only input and output buffers; a C host without a
// device allocator of its own, where a cudaMalloc on every step would also
// synchronise the device.  For them this file keeps the split-context
// scratch (the per-partition partial results) in one file-scope device array
// of fixed size, which every GPU that loads the library holds until the
// process exits, and offers pkv_paged_attention_decode_noalloc, which runs
// the same kernels as pkv_paged_attention_decode on that array.
#include <cuda_runtime.h>

#include <mutex>

#include "pkv_internal.h"

namespace pkv {
namespace {

// The shared scratch.  Host code must not pass this name to a kernel: on the
// host it is only a stand-in for the symbol; the device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_decode_scratch[PKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_decode_scratch on the current device (looked up once per
// device, with that device current).  Returns cudaSuccess and sets *out.
cudaError_t scratch_address(void** out) {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_paged_attention_decode_noalloc(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* context_lens, void* out, int64_t num_seqs, int64_t num_q_heads,
    int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks, int64_t block_size,
    int64_t max_blocks_per_seq, int32_t kv_dtype, int32_t out_dtype, float scale,
    int32_t partition_tokens, uint32_t flags, int32_t* device_error, void* stream) {
    set_last_error("");
    const size_t need = pkv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                  max_blocks_per_seq, block_size, kv_dtype,
                                                  partition_tokens);
    if (need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) {
        set_last_error(
            "these shapes need %zu bytes of split-context scratch but the built-in scratch holds "
            "%zu; pass a larger partition_tokens or use pkv_paged_attention_decode with a "
            "workspace",
            need, (size_t)PKV_NOALLOC_SCRATCH_BYTES);
        return PKV_ERR_WORKSPACE;
    }
    void* scratch = nullptr;
    if (need > 0) {
        cudaError_t e = scratch_address(&scratch);
        if (e != cudaSuccess) {
            set_last_error("cudaGetSymbolAddress of the built-in scratch: %s",
                           cudaGetErrorString(e));
            return PKV_ERR_CUDA;
        }
    }
    // The scheduler counters at the head of the scratch start at zero (device
    // statics are zero-initialised when the module loads) and every call
    // leaves them zero; every partial that a call reads was written earlier
    // in the same call.
    return pkv_paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, out,
                                      scratch, need > 0 ? (size_t)PKV_NOALLOC_SCRATCH_BYTES : 0,
                                      num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                                      block_size, max_blocks_per_seq, kv_dtype, out_dtype, scale,
                                      partition_tokens, flags, device_error, stream);
}
