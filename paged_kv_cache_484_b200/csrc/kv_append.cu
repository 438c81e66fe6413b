// kv_append.cu -- RoPE on the new tokens' q and k, and the k/v write into the
// paged cache slot ("warpllama", Milestones: static KV cache + single-token
// decode, fused RoPE; "Inference From Scratch", ch. 10: block tables), into a
// bf16 / fp32 cache or an 8-bit (E4M3 code x per-tensor scale) one
// ("Efficient LLM Inference", Quantization: rounding to a small set of levels).
//
// One CTA per token; every thread owns one 16-byte chunk of work:
//   * a q or k chunk pair: elements [c*E, c*E+E) of the low half of a head row
//     and the matching elements of the high half (E = 8 bf16 or 4 fp32), i.e.
//     E rotation pairs (x[i], x[i + d/2]);
//   * or one 16-byte chunk of a v row (a bit copy).
// All global loads are issued first; while they are in flight the first d/2
// threads compute sin and cos of the angles pos * theta^(-2i/d) in fp64 (the
// frequencies come from the host, computed with the same fp64 pow as the
// oracle).  Each pair is rotated in fp64 and rounded once to the storage
// type, so the bf16 result is the correctly rounded rotation except in rare
// ties at fp64's last bit.  The kernel moves a few KiB per token and is
// latency bound: one dependent round trip to memory.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int kAppendThreadsMax = 1024;

struct RopeFreq {
    double f[64];  // theta^(-2i/d), i < d/2
};

struct AppendParams {
    void* q;
    const void* k_new;
    const void* v_new;
    const int64_t* positions;
    const int64_t* slot_mapping;
    void* k_cache;
    void* v_cache;
    int Hq, Hkv;
    int64_t num_slots;
    int32_t* err;
    double k_scale, v_scale;  // 8-bit cache only
};

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& v, double (&x)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& v, double (&x)[4]) {
    x[0] = __uint_as_float(v.x);
    x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z);
    x[3] = __uint_as_float(v.w);
}
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& v, double (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        x[2 * k] = bf16lo(w[k]);
        x[2 * k + 1] = bf16hi(w[k]);
    }
}

template <typename T>
__device__ __forceinline__ uint4 pack16(const double (&x)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ uint4 pack16<float>(const double (&x)[4]) {
    return make_uint4(__float_as_uint(__double2float_rn(x[0])), __float_as_uint(__double2float_rn(x[1])),
                      __float_as_uint(__double2float_rn(x[2])), __float_as_uint(__double2float_rn(x[3])));
}
template <>
__device__ __forceinline__ uint4 pack16<__nv_bfloat16>(const double (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
        w[k] = (uint32_t)double_to_bf16_bits(x[2 * k]) |
               ((uint32_t)double_to_bf16_bits(x[2 * k + 1]) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename T, int D>
__global__ void __launch_bounds__(kAppendThreadsMax) kv_append_kernel(
    const __grid_constant__ AppendParams p, const __grid_constant__ RopeFreq fr) {
    constexpr int E = 16 / (int)sizeof(T);  // elements per 16-byte chunk
    constexpr int HALF = D / 2;
    constexpr int CPH = HALF / E;           // chunks per half row
    __shared__ double s_cos[HALF], s_sin[HALF];

    grid_launch_dependents();
    grid_dependency_wait();

    const int64_t t = blockIdx.x;
    const int nq = p.Hq * CPH, nk = p.Hkv * CPH, nv = p.Hkv * 2 * CPH;
    const int total = nq + nk + nv;
    const int64_t slot = p.slot_mapping[t];
    const int64_t pos = p.positions[t];
    const bool write_kv = slot >= 0 && slot < p.num_slots;
    if (slot >= p.num_slots && threadIdx.x == 0) report_error(p.err, PKV_DEVERR_SLOT);
    const int64_t blk = write_kv ? slot / kPageRows : 0;
    const int64_t row = write_kv ? slot % kPageRows : 0;
    T* q = static_cast<T*>(p.q);
    const T* kn = static_cast<const T*>(p.k_new);
    const T* vn = static_cast<const T*>(p.v_new);
    T* kc = static_cast<T*>(p.k_cache);
    T* vc = static_cast<T*>(p.v_cache);

    // Source and destination of work unit `idx` (one 16-byte chunk or pair).
    auto locate = [&](int idx, const T*& src, T*& dst, int& c, bool& is_v) {
        is_v = false;
        if (idx < nq) {
            const int h = idx / CPH;
            c = idx % CPH;
            dst = q + (t * p.Hq + h) * D;
            src = dst;
        } else if (idx < nq + nk) {
            const int j = idx - nq, h = j / CPH;
            c = j % CPH;
            src = kn + (t * p.Hkv + h) * D;
            dst = kc + ((blk * p.Hkv + h) * kPageRows + row) * D;
        } else {
            const int j = idx - nq - nk, h = j / (2 * CPH);
            c = j % (2 * CPH);
            src = vn + (t * p.Hkv + h) * D;
            dst = vc + ((blk * p.Hkv + h) * kPageRows + row) * D;
            is_v = true;
        }
    };

    // First unit of this thread: issue its loads before the angle math.
    const int idx0 = threadIdx.x;
    const T* src0 = nullptr;
    T* dst0 = nullptr;
    int c0 = 0;
    bool v0 = false;
    uint4 lo0 = make_uint4(0, 0, 0, 0), hi0 = lo0;
    // the source rows never depend on the slot, so their loads go out together
    // with the position and slot loads; only the cache stores wait for the slot
    if (idx0 < total) {
        locate(idx0, src0, dst0, c0, v0);
        lo0 = *reinterpret_cast<const uint4*>(src0 + c0 * E);
        if (!v0) hi0 = *reinterpret_cast<const uint4*>(src0 + HALF + c0 * E);
    }
    const bool live0 = idx0 < total && (idx0 < nq || write_kv);
    for (int i = threadIdx.x; i < HALF; i += blockDim.x) {
        double s, c;
        sincos(reduce_two_pi((double)pos * fr.f[i]), &s, &c);
        s_cos[i] = c;
        s_sin[i] = s;
    }
    __syncthreads();

    auto finish = [&](const T* src, T* dst, int c, bool is_v, const uint4& lo, const uint4& hi) {
        if (is_v) {
            *reinterpret_cast<uint4*>(dst + c * E) = lo;
            return;
        }
        double x0[E], x1[E], y0[E], y1[E];
        unpack16<T>(lo, x0);
        unpack16<T>(hi, x1);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const double cs = s_cos[c * E + e], sn = s_sin[c * E + e];
            y0[e] = x0[e] * cs - x1[e] * sn;
            y1[e] = x1[e] * cs + x0[e] * sn;
        }
        *reinterpret_cast<uint4*>(dst + c * E) = pack16<T>(y0);
        *reinterpret_cast<uint4*>(dst + HALF + c * E) = pack16<T>(y1);
    };
    if (live0) finish(src0, dst0, c0, v0, lo0, hi0);
    // Rows wider than one CTA (very many heads): the remaining units.
    for (int idx = idx0 + blockDim.x; idx < total; idx += blockDim.x) {
        if (idx >= nq && !write_kv) break;
        const T* src;
        T* dst;
        int c;
        bool is_v;
        locate(idx, src, dst, c, is_v);
        const uint4 lo = *reinterpret_cast<const uint4*>(src + c * E);
        const uint4 hi = is_v ? lo : *reinterpret_cast<const uint4*>(src + HALF + c * E);
        finish(src, dst, c, is_v, lo, hi);
    }
}

// The same append into the 8-bit cache: q as above; k and v become E4M3
// codes of binary32(x / scale) (x / scale in fp64, then one rounding to
// binary32, then cvt.rn.satfinite to E4M3), k rows into the [16][D] K half
// of the page, v into column `row` of its transposed [D][16] V half (a page
// is one [K | V] region of 2 x 16 D bytes).
template <typename T, int D>
__global__ void __launch_bounds__(kAppendThreadsMax) kv_append_e4m3_kernel(
    const __grid_constant__ AppendParams p, const __grid_constant__ RopeFreq fr) {
    constexpr int E = 16 / (int)sizeof(T);
    constexpr int HALF = D / 2;
    constexpr int CPH = HALF / E;
    __shared__ double s_cos[HALF], s_sin[HALF];

    grid_launch_dependents();
    grid_dependency_wait();

    const int64_t t = blockIdx.x;
    const int nq = p.Hq * CPH, nk = p.Hkv * CPH, nv = p.Hkv * 2 * CPH;
    const int total = nq + nk + nv;
    const int64_t slot = p.slot_mapping[t];
    const int64_t pos = p.positions[t];
    const bool write_kv = slot >= 0 && slot < p.num_slots;
    if (slot >= p.num_slots && threadIdx.x == 0) report_error(p.err, PKV_DEVERR_SLOT);
    const int64_t blk = write_kv ? slot / kPageRows : 0;
    const int row = write_kv ? (int)(slot % kPageRows) : 0;
    T* q = static_cast<T*>(p.q);
    const T* kn = static_cast<const T*>(p.k_new);
    const T* vn = static_cast<const T*>(p.v_new);
    uint8_t* page = static_cast<uint8_t*>(p.k_cache);  // [num_blocks, Hkv, 2, 16 D]

    for (int i = threadIdx.x; i < HALF; i += blockDim.x) {
        double s, c;
        sincos(reduce_two_pi((double)pos * fr.f[i]), &s, &c);
        s_cos[i] = c;
        s_sin[i] = s;
    }
    __syncthreads();

    auto code2 = [](double a, double b, double scale) -> uint32_t {
        return e4m3x2_scaled(a, b, scale);
    };
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
        if (idx >= nq && !write_kv) break;
        if (idx < nq + nk) {
            // a rotation unit: E pairs (x[c E + e], x[c E + e + D/2])
            const bool is_q = idx < nq;
            const int j = is_q ? idx : idx - nq;
            const int h = j / CPH, c = j % CPH;
            const T* src = is_q ? q + (t * p.Hq + h) * D : kn + (t * p.Hkv + h) * D;
            double x0[E], x1[E], y0[E], y1[E];
            unpack16<T>(*reinterpret_cast<const uint4*>(src + c * E), x0);
            unpack16<T>(*reinterpret_cast<const uint4*>(src + HALF + c * E), x1);
#pragma unroll
            for (int e = 0; e < E; ++e)
                rope_rotate_f64(x0[e], x1[e], s_cos[c * E + e], s_sin[c * E + e], y0[e], y1[e]);
            if (is_q) {
                T* dst = q + (t * p.Hq + h) * D;
                *reinterpret_cast<uint4*>(dst + c * E) = pack16<T>(y0);
                *reinterpret_cast<uint4*>(dst + HALF + c * E) = pack16<T>(y1);
            } else {
                uint8_t* dst = page + (blk * p.Hkv + h) * (int64_t)(2 * kPageRows * D) + row * D;
                uint32_t w0[E / 4], w1[E / 4];
#pragma unroll
                for (int k = 0; k < E / 4; ++k) {
                    w0[k] = code2(y0[4 * k], y0[4 * k + 1], p.k_scale) |
                            (code2(y0[4 * k + 2], y0[4 * k + 3], p.k_scale) << 16);
                    w1[k] = code2(y1[4 * k], y1[4 * k + 1], p.k_scale) |
                            (code2(y1[4 * k + 2], y1[4 * k + 3], p.k_scale) << 16);
                }
                if constexpr (E == 8) {
                    *reinterpret_cast<uint2*>(dst + c * E) = make_uint2(w0[0], w0[1]);
                    *reinterpret_cast<uint2*>(dst + HALF + c * E) = make_uint2(w1[0], w1[1]);
                } else {
                    *reinterpret_cast<uint32_t*>(dst + c * E) = w0[0];
                    *reinterpret_cast<uint32_t*>(dst + HALF + c * E) = w1[0];
                }
            }
        } else {
            // a v unit: elements [c E, c E + E) of the row, one byte each into
            // the transposed page (dim-major, 16 tokens per dim)
            const int j = idx - nq - nk, h = j / (2 * CPH), c = j % (2 * CPH);
            double x[E];
            unpack16<T>(*reinterpret_cast<const uint4*>(vn + (t * p.Hkv + h) * D + c * E), x);
            uint8_t* dst = page + (blk * p.Hkv + h) * (int64_t)(2 * kPageRows * D) + kPageRows * D + row;
#pragma unroll
            for (int e = 0; e < E; e += 2) {
                const uint32_t w = code2(x[e], x[e + 1], p.v_scale);
                dst[(c * E + e) * kPageRows] = (uint8_t)(w & 0xFFu);
                dst[(c * E + e + 1) * kPageRows] = (uint8_t)(w >> 8);
            }
        }
    }
}

template <typename T, int D>
cudaError_t launch_typed(const AppendArgs& a) {
    constexpr int E = 16 / (int)sizeof(T);
    constexpr int CPH = (D / 2) / E;
    const int total = (int)((a.Hq + a.Hkv) * CPH + a.Hkv * 2 * CPH);
    const int threads = std::min(kAppendThreadsMax, (total + 31) / 32 * 32);
    AppendParams p;
    p.q = a.q;
    p.k_new = a.k_new;
    p.v_new = a.v_new;
    p.positions = a.positions;
    p.slot_mapping = a.slot_mapping;
    p.k_cache = a.k_cache;
    p.v_cache = a.v_cache;
    p.Hq = (int)a.Hq;
    p.Hkv = (int)a.Hkv;
    p.num_slots = a.num_blocks * (int64_t)kPageRows;
    p.err = a.device_error;
    p.k_scale = (double)a.k_scale;
    p.v_scale = (double)a.v_scale;
    RopeFreq fr;
    for (int i = 0; i < 64; ++i) fr.f[i] = i < D / 2 ? std::pow(a.theta, -(2.0 * i) / D) : 0.0;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.num_tokens);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.e4m3) return cudaLaunchKernelEx(&cfg, kv_append_e4m3_kernel<T, D>, p, fr);
    return cudaLaunchKernelEx(&cfg, kv_append_kernel<T, D>, p, fr);
}

}  // namespace

cudaError_t launch_kv_append(const AppendArgs& a) {
    if (a.dtype == PKV_DTYPE_F32)
        return a.D == 64 ? launch_typed<float, 64>(a) : launch_typed<float, 128>(a);
    return a.D == 64 ? launch_typed<__nv_bfloat16, 64>(a) : launch_typed<__nv_bfloat16, 128>(a);
}

}  // namespace pkv
