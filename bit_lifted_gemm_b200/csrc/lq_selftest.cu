// Self-test of the bounded waits: one thread waits on an mbarrier that nothing
// ever arrives on, through the same bounded-wait helper the GEMV and GEMM use.
// When the limit passes, the helper latches LQ_DEV_TIMEOUT in the device status
// word and the kernel returns, so the context stays usable. It exercises the
// failure-reporting path on the device without faulting or hanging anything.
// In the debug build a second self-test trips the bounds check once, with no
// memory access behind it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lq_debug.cuh"
#include "lq_internal.h"
#include "lq_sm100.cuh"

namespace lq {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(unsigned* status, unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        const uint32_t b = sm100::smem_addr(&bar);
        sm100::mbar_init(b, 1);
        sm100::fence_barrier_init();
        sm100::mbar_wait(b, 0, status, limit_ns);  // no arrival: expires after limit_ns
    }
    __syncwarp();
}

#ifdef LQ_DEBUG
// Index 1 of an extent of 1: the check fails, latches its flag and no access follows.
__global__ void bounds_check_kernel() { (void)LQ_IN_BOUNDS(1, 1); }
#endif

}  // namespace

cudaError_t launch_selftest_wait_timeout(unsigned limit_us, unsigned* status, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(status, (unsigned long long)limit_us * 1000ull);
    return cudaGetLastError();
}

cudaError_t launch_selftest_bounds(cudaStream_t st) {
#ifdef LQ_DEBUG
    bounds_check_kernel<<<1, 1, 0, st>>>();
    return cudaGetLastError();
#else
    (void)st;
    return cudaErrorNotSupported;
#endif
}

}  // namespace lq

LQ_DEBUG_FLAG_TAKE(debug_take_selftest)
