// C ABI of the LiftQuant layer (declared in include/lq.h). This file validates
// arguments synchronously, before any launch, and enqueues the kernels on
// the caller's stream. The only device state it owns is one status word per
// device (a module-scope __device__ variable), which bounded waits in the
// kernels set when they give up.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <initializer_list>

#include "lq.h"
#include "lq_internal.h"

namespace {

__device__ unsigned g_lq_status;
__device__ unsigned g_lq_status_read;

// Reads and clears the status word in one atomic step, so that a timeout a
// kernel on another stream latches meanwhile is either returned or kept.
__global__ void status_exchange_kernel() { g_lq_status_read = atomicExch(&g_lq_status, 0u); }

// Makes `dev` current for its lifetime and restores the previous device.
struct DeviceScope {
    int prev = -1;
    bool ok = false;
    explicit DeviceScope(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) return;
        ok = prev == dev || cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceScope() {
        if (ok && prev >= 0) cudaSetDevice(prev);
    }
};

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int from_cuda(cudaError_t e) { return e == cudaSuccess ? LQ_OK : LQ_ERR_CUDA; }

// Host-side fault injection for the error-path tests (no device fault is ever
// made): LQ_FAULT=launch makes every compute entry point return LQ_ERR_CUDA after
// its argument checks, without launching; LQ_FAULT=timeout makes
// lq_get_device_status report LQ_ERR_TIMEOUT without touching the device.
bool fault_is(const char* mode) {
    const char* f = getenv("LQ_FAULT");
    return f && strcmp(f, mode) == 0;
}

// True if kernels may load and store through p as given: device or managed
// memory, or page-locked host memory that unified addressing maps at the same
// address. Pageable host memory and unknown pointers are refused.
bool device_addressable(const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return true;
    return at.type == cudaMemoryTypeHost && at.devicePointer == p;
}

// True if every non-null pointer is device-addressable (see above).
bool all_addressable(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (p && !device_addressable(p)) return false;
    return true;
}

// True if every non-null pointer is device or managed memory (host memory,
// even page-locked, is refused: the kernels read these operands with TMA or
// keep them in L2).
bool all_device(std::initializer_list<const void*> ps) {
    for (const void* p : ps) {
        if (!p) continue;
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) return false;
    }
    return true;
}

// A byte range [p, p + n) that a call reads, or writes.
struct Span {
    const void* p;
    size_t n;
    bool written;
};

// True when a range the call writes shares a byte with another of its ranges:
// an output aliasing an input (or another output) would be read and written by
// different CTAs in no fixed order. Null pointers and empty ranges never overlap;
// sizes come from validated int arguments, so the sums cannot wrap.
bool aliased(std::initializer_list<Span> spans) {
    const Span* v = spans.begin();
    const size_t n = spans.size();
    for (size_t i = 0; i < n; ++i)
        for (size_t j = i + 1; j < n; ++j) {
            if (!(v[i].written || v[j].written) || !v[i].p || !v[j].p || !v[i].n || !v[j].n) continue;
            const uintptr_t a = reinterpret_cast<uintptr_t>(v[i].p), b = reinterpret_cast<uintptr_t>(v[j].p);
            if (a < b + v[j].n && b < a + v[i].n) return true;
        }
    return false;
}

size_t nbytes(long long count, size_t elem) { return (size_t)count * elem; }

// Device address of the status word on the current device (looked up once per device).
unsigned* status_word(int* err) {
    static unsigned* addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) {
        *err = LQ_ERR_CUDA;
        return nullptr;
    }
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_lq_status) != cudaSuccess) {
            *err = LQ_ERR_CUDA;
            return nullptr;
        }
        addr[dev] = static_cast<unsigned*>(p);
    }
    *err = LQ_OK;
    return addr[dev];
}

// 1 if the current device is an sm_100 part, 0 if not, -1 on error (cached per device).
int is_sm100() {
    static signed char cache[kMaxDevices];
    static bool init[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return -1;
    if (!init[dev]) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return -1;
        if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return -1;
        cache[dev] = (major == 10 && minor == 0) ? 1 : 0;
        init[dev] = true;
    }
    return cache[dev];
}

}  // namespace

extern "C" {

const char* lq_status_str(int status) {
    switch (status) {
        case LQ_OK: return "LQ_OK";
        case LQ_ERR_INVALID_ARG: return "LQ_ERR_INVALID_ARG";
        case LQ_ERR_UNSUPPORTED: return "LQ_ERR_UNSUPPORTED";
        case LQ_ERR_CUDA: return "LQ_ERR_CUDA";
        case LQ_ERR_TIMEOUT: return "LQ_ERR_TIMEOUT";
        case LQ_ERR_TOO_LARGE: return "LQ_ERR_TOO_LARGE";
        case LQ_ERR_BOUNDS: return "LQ_ERR_BOUNDS";
        default: return "LQ_ERR_UNKNOWN";
    }
}

int lq_lifted_dim(int in, int d, int D) {
    if (in <= 0 || d <= 0 || D <= 0 || in % d != 0) return -1;
    long long k = (long long)(in / d) * D;
    k = (k + 31) / 32 * 32;
    return k > 0x7fffffffLL ? -1 : (int)k;
}

int lq_pack_signs(const int8_t* signs_pm1, int out, int K, uint32_t* packed, void* stream) {
    if (!signs_pm1 || !packed || !aligned16(signs_pm1) || !aligned16(packed)) return LQ_ERR_INVALID_ARG;
    if (out < 1 || K < 32 || K % 32 != 0) return LQ_ERR_INVALID_ARG;
    if (aliased({{signs_pm1, nbytes((long long)out * K, 1), false}, {packed, nbytes((long long)out * (K / 32), 4), true}}))
        return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    if (!all_device({signs_pm1, packed})) return LQ_ERR_INVALID_ARG;
    return from_cuda(lq::launch_pack(signs_pm1, out, K, packed, static_cast<cudaStream_t>(stream)));
}

int lq_unpack_signs(const uint32_t* packed, int out, int K, int8_t* signs_pm1, void* stream) {
    if (!signs_pm1 || !packed || !aligned16(signs_pm1) || !aligned16(packed)) return LQ_ERR_INVALID_ARG;
    if (out < 1 || K < 32 || K % 32 != 0) return LQ_ERR_INVALID_ARG;
    if (aliased({{packed, nbytes((long long)out * (K / 32), 4), false}, {signs_pm1, nbytes((long long)out * K, 1), true}}))
        return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    if (!all_device({packed, signs_pm1})) return LQ_ERR_INVALID_ARG;
    return from_cuda(lq::launch_unpack(packed, out, K, signs_pm1, static_cast<cudaStream_t>(stream)));
}

int lq_lift_activations(const void* a, int a_dtype, int batch, int in, const float* tinv, int tblk,
                        const float* M, int d, int D, void* u, int u_dtype, int K, void* stream) {
    if (!a || !M || !u || !aligned16(a) || !aligned16(M) || !aligned16(u)) return LQ_ERR_INVALID_ARG;
    if (tinv && !aligned16(tinv)) return LQ_ERR_INVALID_ARG;
    if ((a_dtype != LQ_F32 && a_dtype != LQ_BF16) || (u_dtype != LQ_F32 && u_dtype != LQ_BF16))
        return LQ_ERR_INVALID_ARG;
    if (batch < 1 || in < 1 || d < 1 || d > 64 || D < 1 || D > 256 || d * D > 4096) return LQ_ERR_INVALID_ARG;
    if (lq_lifted_dim(in, d, D) != K) return LQ_ERR_INVALID_ARG;
    if (tinv && (tblk < 1 || tblk > 256 || in % tblk != 0)) return LQ_ERR_INVALID_ARG;
    if (aliased({{a, nbytes((long long)batch * in, a_dtype == LQ_BF16 ? 2 : 4), false},
                 {tinv, tinv ? nbytes((long long)in * tblk, 4) : 0, false},
                 {M, nbytes((long long)d * D, 4), false},
                 {u, nbytes((long long)batch * K, u_dtype == LQ_BF16 ? 2 : 4), true}}))
        return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    const int sm = is_sm100();
    if (sm < 0) return LQ_ERR_CUDA;
    if (sm == 0) return LQ_ERR_UNSUPPORTED;
    if (!all_device({a, tinv, M, u})) return LQ_ERR_INVALID_ARG;
    int err = LQ_OK;
    unsigned* status = status_word(&err);
    if (!status) return err;
    return from_cuda(lq::launch_lift(a, a_dtype == LQ_BF16, batch, in, tinv, tblk, M, d, D, u, u_dtype == LQ_BF16,
                                     K, status, static_cast<cudaStream_t>(stream)));
}

int lq_lift_activations_kron(const void* a, int a_dtype, int batch, int in, const float* r1, const float* q1,
                             int n1, const float* q2, int n2, const float* r2, const float* M, int d, int D,
                             void* u, int u_dtype, int K, void* stream) {
    if (!a || !q1 || !q2 || !M || !u) return LQ_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(q1) || !aligned16(q2) || !aligned16(M) || !aligned16(u))
        return LQ_ERR_INVALID_ARG;
    if ((r1 && !aligned16(r1)) || (r2 && !aligned16(r2))) return LQ_ERR_INVALID_ARG;
    if ((a_dtype != LQ_F32 && a_dtype != LQ_BF16) || (u_dtype != LQ_F32 && u_dtype != LQ_BF16))
        return LQ_ERR_INVALID_ARG;
    if (batch < 1 || in < 1 || in > 16384 || d < 1 || d > 64 || D < 1 || D > 256 || d * D > 4096)
        return LQ_ERR_INVALID_ARG;
    if (n1 < 1 || n1 > 256 || n2 < 1 || n2 > 128 || n1 * n2 != in || in % d != 0) return LQ_ERR_INVALID_ARG;
    if (lq_lifted_dim(in, d, D) != K) return LQ_ERR_INVALID_ARG;
    if (!lq::lift_kron_supported(batch, in, n1, n2, d, D)) return LQ_ERR_INVALID_ARG;
    if (aliased({{a, nbytes((long long)batch * in, a_dtype == LQ_BF16 ? 2 : 4), false},
                 {r1, nbytes(in, 4), false},
                 {q1, nbytes((long long)n1 * n1, 4), false},
                 {q2, nbytes((long long)n2 * n2, 4), false},
                 {r2, nbytes(in / d, 4), false},
                 {M, nbytes((long long)d * D, 4), false},
                 {u, nbytes((long long)batch * K, u_dtype == LQ_BF16 ? 2 : 4), true}}))
        return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    const int sm = is_sm100();
    if (sm < 0) return LQ_ERR_CUDA;
    if (sm == 0) return LQ_ERR_UNSUPPORTED;
    if (!all_device({a, r1, q1, q2, r2, M, u})) return LQ_ERR_INVALID_ARG;
    if (lq::lift_kron_tc_supported(a_dtype == LQ_BF16, u_dtype == LQ_BF16, batch, in, n1, n2, d, D, K)) {
        // prefill: both products on the tensor cores
        int err = LQ_OK;
        unsigned* status = status_word(&err);
        if (!status) return err;
        return from_cuda(lq::launch_lift_kron_tc(static_cast<const uint16_t*>(a), batch, in, r1, q1, n1, q2, n2, r2, M,
                                                 d, D, u, K, status, static_cast<cudaStream_t>(stream)));
    }
    return from_cuda(lq::launch_lift_kron(a, a_dtype == LQ_BF16, batch, in, r1, q1, n1, q2, n2, r2, M, d, D, u,
                                          u_dtype == LQ_BF16, K, static_cast<cudaStream_t>(stream)));
}

int lq_encode(const float* w, int rows, int in, const float* M, int d, int D, uint32_t* packed, int K, float* err,
              void* stream) {
    if (!w || !M || !packed || !aligned16(w) || !aligned16(M) || !aligned16(packed)) return LQ_ERR_INVALID_ARG;
    if (err && !aligned16(err)) return LQ_ERR_INVALID_ARG;
    if (rows < 1 || in < 1 || d < 1 || d > 24 || D < d || D > 63 || D - d > 24 || in % d != 0)
        return LQ_ERR_INVALID_ARG;
    if (lq_lifted_dim(in, d, D) != K) return LQ_ERR_INVALID_ARG;
    if (aliased({{w, nbytes((long long)rows * in, 4), false},
                 {M, nbytes((long long)d * D, 4), false},
                 {packed, nbytes((long long)rows * (K / 32), 4), true},
                 {err, err ? nbytes((long long)rows * (in / d), 4) : 0, true}}))
        return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    const int sm = is_sm100();
    if (sm < 0) return LQ_ERR_CUDA;
    if (sm == 0) return LQ_ERR_UNSUPPORTED;
    if (!all_device({w, M, packed, err})) return LQ_ERR_INVALID_ARG;
    return from_cuda(lq::launch_encode(w, rows, in, M, d, D, packed, K, err, static_cast<cudaStream_t>(stream)));
}

int lq_selftest_wait_timeout(unsigned limit_us, void* stream) {
    if (limit_us < 1 || limit_us > 1000000) return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    const int sm = is_sm100();
    if (sm < 0) return LQ_ERR_CUDA;
    if (sm == 0) return LQ_ERR_UNSUPPORTED;
    int err = LQ_OK;
    unsigned* status = status_word(&err);
    if (!status) return err;
    return from_cuda(lq::launch_selftest_wait_timeout(limit_us, status, static_cast<cudaStream_t>(stream)));
}

size_t lq_gemv_workspace_size(int out, int K, int batch) {
    if (out < 1 || K < 32 || K % 32 != 0 || batch < 1 || batch > 16) return 0;
    return lq::gemv_workspace_size(out, K, batch);
}

int lq_gemv(const uint32_t* packed, const float* s, int out, int K, const float* u, int batch, float* o,
            void* workspace, size_t workspace_bytes, void* stream) {
    if (!packed || !s || !u || !o || !workspace) return LQ_ERR_INVALID_ARG;
    if (!aligned16(packed) || !aligned16(s) || !aligned16(u) || !aligned16(o)) return LQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LQ_ERR_INVALID_ARG;
    if (out < 1 || K < 32 || K % 32 != 0 || batch < 1 || batch > 16) return LQ_ERR_INVALID_ARG;
    const size_t need = lq::gemv_workspace_size(out, K, batch);
    if (need == 0 || workspace_bytes < need) return LQ_ERR_INVALID_ARG;
    if (aliased({{packed, nbytes((long long)out * (K / 32), 4), false},
                 {s, nbytes(out, 4), false},
                 {u, nbytes((long long)batch * K, 4), false},
                 {o, nbytes((long long)batch * out, 4), true},
                 {workspace, need, true}}))
        return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    const int sm = is_sm100();
    if (sm < 0) return LQ_ERR_CUDA;
    if (sm == 0) return LQ_ERR_UNSUPPORTED;
    if (!all_device({packed, s, u, o, workspace})) return LQ_ERR_INVALID_ARG;
    int err = LQ_OK;
    unsigned* status = status_word(&err);
    if (!status) return err;
    return from_cuda(lq::launch_gemv(packed, s, out, K, u, batch, o, workspace, status,
                                     static_cast<cudaStream_t>(stream)));
}

int lq_lift_gemv(const void* a, int a_dtype, int batch, int in, const float* tinv, int tblk, const float* M, int d,
                 int D, const uint32_t* packed, const float* s, int out, int K, float* u, float* o,
                 void* workspace, size_t workspace_bytes, void* stream) {
    if (!a || !M || !u || !packed || !s || !o || !workspace) return LQ_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(M) || !aligned16(u) || !aligned16(packed) || !aligned16(s) || !aligned16(o))
        return LQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LQ_ERR_INVALID_ARG;
    if (tinv && !aligned16(tinv)) return LQ_ERR_INVALID_ARG;
    if (a_dtype != LQ_F32 && a_dtype != LQ_BF16) return LQ_ERR_INVALID_ARG;
    if (batch < 1 || batch > 16 || in < 1 || d < 1 || d > 64 || D < 1 || D > 256 || d * D > 4096)
        return LQ_ERR_INVALID_ARG;
    if (lq_lifted_dim(in, d, D) != K) return LQ_ERR_INVALID_ARG;
    if (tinv && (tblk < 1 || tblk > 256 || in % tblk != 0)) return LQ_ERR_INVALID_ARG;
    if (out < 1) return LQ_ERR_INVALID_ARG;
    const size_t need = lq::gemv_workspace_size(out, K, batch);
    if (need == 0 || workspace_bytes < need) return LQ_ERR_INVALID_ARG;
    if (aliased({{a, nbytes((long long)batch * in, a_dtype == LQ_BF16 ? 2 : 4), false},
                 {tinv, tinv ? nbytes((long long)in * tblk, 4) : 0, false},
                 {M, nbytes((long long)d * D, 4), false},
                 {packed, nbytes((long long)out * (K / 32), 4), false},
                 {s, nbytes(out, 4), false},
                 {u, nbytes((long long)batch * K, 4), true},
                 {o, nbytes((long long)batch * out, 4), true},
                 {workspace, need, true}}))
        return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    const int sm = is_sm100();
    if (sm < 0) return LQ_ERR_CUDA;
    if (sm == 0) return LQ_ERR_UNSUPPORTED;
    if (!all_addressable({a, o}) || !all_device({tinv, M, packed, s, u, workspace})) return LQ_ERR_INVALID_ARG;
    int err = LQ_OK;
    unsigned* status = status_word(&err);
    if (!status) return err;
    return from_cuda(lq::launch_lift_gemv(a, a_dtype == LQ_BF16, batch, in, tinv, tblk, M, d, D, packed, s, out, K, u,
                                          o, workspace, status, static_cast<cudaStream_t>(stream)));
}

int lq_gemm(const uint32_t* packed, const float* s, int out, int K, const uint16_t* u_bf16, int tokens, float* o,
            void* stream) {
    if (!packed || !s || !u_bf16 || !o) return LQ_ERR_INVALID_ARG;
    if (!aligned16(packed) || !aligned16(s) || !aligned16(u_bf16) || !aligned16(o)) return LQ_ERR_INVALID_ARG;
    if (out < 1 || K < 32 || K % 32 != 0 || tokens < 1) return LQ_ERR_INVALID_ARG;
    if (aliased({{packed, nbytes((long long)out * (K / 32), 4), false},
                 {s, nbytes(out, 4), false},
                 {u_bf16, nbytes((long long)tokens * K, 2), false},
                 {o, nbytes((long long)tokens * out, 4), true}}))
        return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    const int sm = is_sm100();
    if (sm < 0) return LQ_ERR_CUDA;
    if (sm == 0) return LQ_ERR_UNSUPPORTED;
    if (!all_device({packed, s, u_bf16, o})) return LQ_ERR_INVALID_ARG;
    int err = LQ_OK;
    unsigned* status = status_word(&err);
    if (!status) return err;
    return from_cuda(lq::launch_gemm(packed, s, out, K, u_bf16, tokens, o, status, static_cast<cudaStream_t>(stream)));
}

int lq_get_device_status(void* stream) {
    if (fault_is("timeout")) return LQ_ERR_TIMEOUT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0;
    if (cudaStreamGetDevice(st, &dev) != cudaSuccess) return LQ_ERR_CUDA;
    DeviceScope scope(dev);  // the status word of the stream's device
    if (!scope.ok) return LQ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return LQ_ERR_CUDA;
    status_exchange_kernel<<<1, 1, 0, st>>>();
    if (cudaGetLastError() != cudaSuccess) return LQ_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_lq_status_read, sizeof(v), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return LQ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return LQ_ERR_CUDA;
#ifdef LQ_DEBUG
    // every file's flag is read and cleared, whichever is set
    const unsigned bounds = lq::debug_take_gemm() | lq::debug_take_lift() | lq::debug_take_lift_kron() |
                            lq::debug_take_lift_tc() | lq::debug_take_lift_kron_tc() | lq::debug_take_encode() |
                            lq::debug_take_pack() | lq::debug_take_selftest();
    if (bounds) return LQ_ERR_BOUNDS;
#endif
    return (v & LQ_DEV_TIMEOUT) ? LQ_ERR_TIMEOUT : LQ_OK;
}

int lq_selftest_bounds(void* stream) {
#ifdef LQ_DEBUG
    if (fault_is("launch")) return LQ_ERR_CUDA;
    const int sm = is_sm100();
    if (sm < 0) return LQ_ERR_CUDA;
    if (sm == 0) return LQ_ERR_UNSUPPORTED;
    return from_cuda(lq::launch_selftest_bounds(static_cast<cudaStream_t>(stream)));
#else
    (void)stream;
    return LQ_ERR_UNSUPPORTED;
#endif
}

int lq_is_debug_build(void) {
#ifdef LQ_DEBUG
    return 1;
#else
    return 0;
#endif
}

// ---------------------------------------------------------------- decode GEMV without allocation
//
// For callers that cannot allocate device memory (see lq.h): the scratch that
// lq_gemv takes as a workspace lives in this fixed device array instead. Every
// device that loads the library holds it until the process exits. Its address is
// looked up once per device, with that device current; host code must never hand
// the array's name itself to a kernel (on the host it is only a stand-in).

}  // extern "C"

static __device__ __align__(256) uint8_t g_lq_static_scratch[LQ_GEMV_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the static scratch on the current device, or null on error.
void* static_scratch() {
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return nullptr;
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_lq_static_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

int lq_gemv_noalloc(const uint32_t* packed, const float* s, int out, int K, const float* u, int batch, float* o,
                    void* stream) {
    if (!packed || !s || !u || !o) return LQ_ERR_INVALID_ARG;
    if (!aligned16(packed) || !aligned16(s) || !aligned16(u) || !aligned16(o)) return LQ_ERR_INVALID_ARG;
    if (out < 1 || K < 32 || K % 32 != 0 || batch < 1 || batch > 16) return LQ_ERR_INVALID_ARG;
    const size_t need = lq::gemv_workspace_size(out, K, batch);
    if (need == 0) return LQ_ERR_INVALID_ARG;
    if (need > LQ_GEMV_NOALLOC_SCRATCH_BYTES) return LQ_ERR_TOO_LARGE;
    if (aliased({{packed, nbytes((long long)out * (K / 32), 4), false},
                 {s, nbytes(out, 4), false},
                 {u, nbytes((long long)batch * K, 4), false},
                 {o, nbytes((long long)batch * out, 4), true}}))
        return LQ_ERR_INVALID_ARG;
    if (fault_is("launch")) return LQ_ERR_CUDA;
    const int sm = is_sm100();
    if (sm < 0) return LQ_ERR_CUDA;
    if (sm == 0) return LQ_ERR_UNSUPPORTED;
    if (!all_device({packed, s, u, o})) return LQ_ERR_INVALID_ARG;
    void* scratch = static_scratch();
    if (!scratch) return LQ_ERR_CUDA;
    int err = LQ_OK;
    unsigned* status = status_word(&err);
    if (!status) return err;
    return from_cuda(lq::launch_gemv(packed, s, out, K, u, batch, o, scratch, status,
                                     static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
