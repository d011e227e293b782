// Device-side bounds checks of the debug build (liblq_debug.so, compiled with
// -DLQ_DEBUG): every guarded global load or store first tests its element index
// against the extent of its buffer, as computed from the call's arguments. A
// failed test sets this file's flag and the access is skipped. Nothing traps or
// faults. lq_get_device_status then reports LQ_ERR_BOUNDS. In the release build
// the checks compile to `true` and cost nothing.
//
// Each .cu file that includes this header gets its own flag (a static device
// variable: the library is compiled without relocatable device code) and must
// define its take-and-clear function once with LQ_DEBUG_FLAG_TAKE(name), which
// lq_api.cu calls through lq_internal.h.
#pragma once

#include <cuda_runtime.h>

#ifdef LQ_DEBUG

static __device__ unsigned g_lq_bounds_flag;

// True when 0 <= i < n; otherwise records the violation and returns false.
__device__ __forceinline__ bool lq_in_bounds(long long i, long long n) {
    const bool ok = i >= 0 && i < n;
    if (!ok) atomicOr(&g_lq_bounds_flag, 1u);
    return ok;
}
#define LQ_IN_BOUNDS(i, n) lq_in_bounds((long long)(i), (long long)(n))

// Host: read and clear this file's flag (non-zero after a failed check).
#define LQ_DEBUG_FLAG_TAKE(name)                                                              \
    namespace lq {                                                                           \
    unsigned name() {                                                                        \
        unsigned v = 0, z = 0;                                                               \
        if (cudaMemcpyFromSymbol(&v, g_lq_bounds_flag, sizeof(v)) != cudaSuccess) return 0u; \
        cudaMemcpyToSymbol(g_lq_bounds_flag, &z, sizeof(z));                                 \
        return v;                                                                            \
    }                                                                                        \
    }

#else

#define LQ_IN_BOUNDS(i, n) true
#define LQ_DEBUG_FLAG_TAKE(name)

#endif
