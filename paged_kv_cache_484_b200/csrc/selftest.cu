// selftest.cu -- the bounded in-kernel wait, run until it gives up.
//
// Every pipeline wait of the decode and prefill kernels goes through
// mbar_wait_for (pkv_device.cuh).  This kernel waits on a shared-memory
// barrier that nothing ever arrives on, with a caller-given limit, so the
// give-up path (PKV_DEVERR_TIMEOUT, then a normal return) runs on the GPU
// without any real stage being starved.  No copy is in flight on the barrier,
// so the kernel may exit as soon as the wait returns.
#include <cuda_runtime.h>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

__global__ void __launch_bounds__(32) bounded_wait_kernel(uint64_t limit_ns, int32_t* err,
                                                          uint64_t* waited_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) mbar_init(&bar, 1);  // one arrival would complete it; none comes
    fence_barrier_init();
    __syncwarp();
    if (threadIdx.x != 0) return;
    const uint64_t t0 = global_timer_ns();
    const bool done = mbar_wait_for(&bar, 0, limit_ns);
    const uint64_t t1 = global_timer_ns();
    if (!done) report_error(err, PKV_DEVERR_TIMEOUT);
    if (waited_ns) *waited_ns = t1 - t0;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_selftest_bounded_wait(uint32_t limit_us, int32_t* device_error,
                                                uint64_t* waited_ns, void* stream) {
    set_last_error("");
    if (limit_us == 0 || limit_us > 2000000u) {
        set_last_error("limit_us must be in [1, 2000000], got %u", limit_us);
        return PKV_ERR_INVALID_ARG;
    }
    if (!device_error) {
        set_last_error("device_error is required");
        return PKV_ERR_INVALID_ARG;
    }
    bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        (uint64_t)limit_us * 1000ull, device_error, waited_ns);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_last_error("bounded-wait self-test launch: %s", cudaGetErrorString(e));
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

extern "C" pkv_status pkv_get_device_error(const int32_t* device_error, void* stream,
                                           int32_t* code_out) {
    set_last_error("");
    if (!device_error || !code_out) {
        set_last_error("device_error and code_out are required");
        return PKV_ERR_INVALID_ARG;
    }
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, device_error, sizeof(v), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        set_last_error("reading the device error word: %s", cudaGetErrorString(e));
        return PKV_ERR_CUDA;
    }
    *code_out = v;
    if (v != 0) {
        set_last_error("device error word %#x:%s%s%s%s%s", (unsigned)v,
                       (v & PKV_DEVERR_SLOT) ? " slot" : "",
                       (v & PKV_DEVERR_BLOCK_ID) ? " block_id" : "",
                       (v & PKV_DEVERR_CONTEXT_LEN) ? " context_len" : "",
                       (v & PKV_DEVERR_TIMEOUT) ? " timeout" : "",
                       (v & PKV_DEVERR_PREFIX) ? " prefix" : "");
        return PKV_ERR_DEVICE;
    }
    return PKV_OK;
}
