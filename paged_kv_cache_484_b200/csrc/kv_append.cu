// kv_append.cu -- RoPE on the new tokens' q and k, and the k/v write into the
// paged cache slot ("warpllama", Milestones: static KV cache + single-token
// decode, fused RoPE; "Inference From Scratch", ch. 10: block tables).
//
// One CTA per token.  The d/2 rotation angles pos * theta^(-2i/d) and their
// sines and cosines are computed once per token in fp64; each pair
// (x[i], x[i + d/2]) is rotated in fp64 and rounded once to the storage type,
// so the bf16 result is the correctly rounded rotation whenever the fp64
// sine/cosine are within half an fp64 ulp of the truth.  v is copied with
// 16-byte vector moves.  The kernel is memory-trivial (a few KiB per token).
#include <cuda_bf16.h>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

template <typename T>
__device__ __forceinline__ double load_d(const T* p);
template <>
__device__ __forceinline__ double load_d<float>(const float* p) {
    return (double)*p;
}
template <>
__device__ __forceinline__ double load_d<__nv_bfloat16>(const __nv_bfloat16* p) {
    return (double)__bfloat162float(*p);
}

template <typename T>
__device__ __forceinline__ void store_d(T* p, double v);
template <>
__device__ __forceinline__ void store_d<float>(float* p, double v) {
    *p = __double2float_rn(v);
}
template <>
__device__ __forceinline__ void store_d<__nv_bfloat16>(__nv_bfloat16* p, double v) {
    *reinterpret_cast<uint16_t*>(p) = double_to_bf16_bits(v);
}

template <typename T, int D>
__global__ void __launch_bounds__(128) kv_append_kernel(
    T* __restrict__ q, const T* __restrict__ k_new, const T* __restrict__ v_new,
    const int64_t* __restrict__ positions, const int64_t* __restrict__ slot_mapping,
    T* __restrict__ k_cache, T* __restrict__ v_cache, int Hq, int Hkv, int64_t num_slots,
    double theta, int32_t* __restrict__ device_error) {
    constexpr int HALF = D / 2;
    __shared__ double s_cos[HALF], s_sin[HALF];

    grid_launch_dependents();
    grid_dependency_wait();

    const int64_t t = blockIdx.x;
    const int64_t pos = positions[t];
    for (int i = threadIdx.x; i < HALF; i += blockDim.x) {
        const double freq = pow(theta, -(2.0 * (double)i) / (double)D);
        double s, c;
        sincos((double)pos * freq, &s, &c);
        s_cos[i] = c;
        s_sin[i] = s;
    }
    __syncthreads();

    const int64_t slot = slot_mapping[t];
    const bool write_kv = slot >= 0 && slot < num_slots;
    if (slot >= num_slots && threadIdx.x == 0) report_error(device_error, PKV_DEVERR_SLOT);
    const int64_t blk = write_kv ? slot / kPageRows : 0;
    const int64_t row = write_kv ? slot % kPageRows : 0;

    // q: all heads, in place.  k: rotated into the cache row.
    const int qpairs = Hq * HALF;
    const int kpairs = write_kv ? Hkv * HALF : 0;
    for (int idx = threadIdx.x; idx < qpairs + kpairs; idx += blockDim.x) {
        const T* src;
        T* dst;
        int i;
        if (idx < qpairs) {
            const int h = idx / HALF;
            i = idx % HALF;
            dst = q + (t * Hq + h) * D;
            src = dst;
        } else {
            const int j = idx - qpairs;
            const int h = j / HALF;
            i = j % HALF;
            src = k_new + (t * Hkv + h) * D;
            dst = k_cache + ((blk * Hkv + h) * kPageRows + row) * D;
        }
        const double x0 = load_d(src + i), x1 = load_d(src + i + HALF);
        const double c = s_cos[i], s = s_sin[i];
        store_d(dst + i, x0 * c - x1 * s);
        store_d(dst + i + HALF, x1 * c + x0 * s);
    }

    // v: bit copy, 16 bytes per thread-step.
    if (write_kv) {
        constexpr int VEC = 16 / sizeof(T);
        constexpr int ROW_VECS = D / VEC;
        const int n = Hkv * ROW_VECS;
        for (int idx = threadIdx.x; idx < n; idx += blockDim.x) {
            const int h = idx / ROW_VECS, c = idx % ROW_VECS;
            const uint4* s4 = reinterpret_cast<const uint4*>(v_new + (t * Hkv + h) * D) + c;
            uint4* d4 =
                reinterpret_cast<uint4*>(v_cache + ((blk * Hkv + h) * kPageRows + row) * D) + c;
            *d4 = *s4;
        }
    }
}

template <typename T, int D>
cudaError_t launch_typed(const AppendArgs& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.num_tokens);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kv_append_kernel<T, D>, static_cast<T*>(a.q),
                              static_cast<const T*>(a.k_new), static_cast<const T*>(a.v_new),
                              a.positions, a.slot_mapping, static_cast<T*>(a.k_cache),
                              static_cast<T*>(a.v_cache), (int)a.Hq, (int)a.Hkv,
                              a.num_blocks * (int64_t)kPageRows, a.theta, a.device_error);
}

}  // namespace

cudaError_t launch_kv_append(const AppendArgs& a) {
    if (a.dtype == PKV_DTYPE_F32)
        return a.D == 64 ? launch_typed<float, 64>(a) : launch_typed<float, 128>(a);
    return a.D == 64 ? launch_typed<__nv_bfloat16, 64>(a) : launch_typed<__nv_bfloat16, 128>(a);
}

}  // namespace pkv
