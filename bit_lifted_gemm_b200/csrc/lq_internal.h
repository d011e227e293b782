// Internal launchers of the LiftQuant sm_100a kernels. Each returns the
// cudaError_t of its launch; argument validation happens in lq_api.cu before
// any of these is called.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

// Bits of the device status word (read and cleared by lq_get_device_status).
#define LQ_DEV_TIMEOUT 1u

namespace lq {

cudaError_t launch_pack(const int8_t* signs, int out, int K, uint32_t* packed, cudaStream_t st);
cudaError_t launch_unpack(const uint32_t* packed, int out, int K, int8_t* signs, cudaStream_t st);

// Activation lift u = blockdiag(M^T) T^{-1} a. `status` is the device status word
// (the tensor-core prefill variant has bounded waits).
cudaError_t launch_lift(const void* a, bool a_bf16, int batch, int in, const float* tinv, int tblk,
                        const float* M, int d, int D, void* u, bool u_bf16, int K, unsigned* status,
                        cudaStream_t st);

// Prefill lift with the whitening on tcgen05 (bf16 activations, 128-wide
// whitening blocks, at least 64 tokens); launch_lift dispatches to it.
bool lift_tc_supported(bool a_bf16, int batch, int in, const float* tinv, int tblk, int d, int D);
cudaError_t launch_lift_tc(const uint16_t* a, int batch, int in, const float* tinv, const float* M, int d, int D,
                           void* u, bool u_bf16, int K, unsigned* status, cudaStream_t st);

// Lift with a Kronecker-factored whitening T^{-1} = diag(r2) (Q1 kron Q2) diag(r1)
// as (Q1 X) Q2^T, each CTA owning a slice of rows of the result.
// lift_kron_supported tells whether the shapes fit its shared-memory plan.
bool lift_kron_supported(int batch, int in, int n1, int n2, int d, int D);
cudaError_t launch_lift_kron(const void* a, bool a_bf16, int batch, int in, const float* r1, const float* q1,
                             int n1, const float* q2, int n2, const float* r2, const float* M, int d, int D,
                             void* u, bool u_bf16, int K, cudaStream_t st);

// The same lift for prefill on tcgen05 (lq_lift_kron_tc.cu): bf16 activations
// and u, at least 64 tokens, n1 <= 64, n2 a multiple of 16 up to 128, d <= 16
// dividing n2, D >= 2 d a multiple of 4 (u's rows hold the intermediate product first).
bool lift_kron_tc_supported(bool a_bf16, bool u_bf16, int batch, int in, int n1, int n2, int d, int D, int K);
cudaError_t launch_lift_kron_tc(const uint16_t* a, int batch, int in, const float* r1, const float* q1, int n1,
                                const float* q2, int n2, const float* r2, const float* M, int d, int D, void* u,
                                int K, unsigned* status, cudaStream_t st);

// Encoder (offline): nearest lifted codewords of weight blocks by the
// pseudo-inverse start plus the 2^{D-d} auxiliary-vector search, float64,
// written as packed signs. encode_smem gives its shared-memory need.
size_t encode_smem(int d, int D);
cudaError_t launch_encode(const float* w, int rows, int in, const float* M, int d, int D, uint32_t* packed, int K,
                          float* err, cudaStream_t st);

// Self-test of the bounded waits: one wait that nothing completes, limit_us long.
cudaError_t launch_selftest_wait_timeout(unsigned limit_us, unsigned* status, cudaStream_t st);
// Debug build: one failed bounds check with no access behind it (cudaErrorNotSupported in release).
cudaError_t launch_selftest_bounds(cudaStream_t st);

#ifdef LQ_DEBUG
// Debug build: read and clear the bounds flag of each source file (non-zero after
// a failed check), on the current device.
unsigned debug_take_gemm();
unsigned debug_take_lift();
unsigned debug_take_lift_kron();
unsigned debug_take_lift_tc();
unsigned debug_take_lift_kron_tc();
unsigned debug_take_encode();
unsigned debug_take_pack();
unsigned debug_take_selftest();
#endif

// Decode GEMV (lq_decode.h): the quantizer writes u's digit planes into the
// caller's workspace, then the mma.sync kernel (batch 1..2, or when the
// tcgen05 plan does not fit) or the tcgen05 kernel (batch >= 3) contracts.
// `status` is the device status word that bounded waits report to.
// gemv_workspace_size is 0 when no launch plan fits the shape (each mma.sync
// CTA keeps 64-bit partial sums for its rows, so a very large `out` does not fit).
size_t gemv_workspace_size(int out, int K, int batch);
cudaError_t launch_gemv(const uint32_t* packed, const float* s, int out, int K, const float* u,
                        int batch, float* o, void* ws, unsigned* status, cudaStream_t st);

// Decode step: the lift into u, the quantizer, then the contraction, each a
// programmatic dependent of the one before.
cudaError_t launch_lift_gemv(const void* a, bool a_bf16, int batch, int in, const float* tinv, int tblk,
                             const float* M, int d, int D, const uint32_t* packed, const float* s, int out, int K,
                             float* u, float* o, void* ws, unsigned* status, cudaStream_t st);

struct DecodePlan;
// The quantizers (lq_quant.cu): 32-bit fixed point for the mma.sync kernel
// (it also clears `nzero` words at `zero`), block-scaled e2m1 digits for the
// tcgen05 kernel (it also clears the kernel's group counters).
cudaError_t launch_quant_mx(const float* u, const DecodePlan& p, void* ws, cudaStream_t st);
// The tcgen05 contraction (lq_gemv_tc.cu): plan_tc fills the tc_* fields and
// returns whether the shape takes that kernel; tc_slot_bytes is the size of its
// partial-sum slots in the workspace.
bool plan_tc(DecodePlan& p);
size_t tc_slot_bytes(const DecodePlan& p);
cudaError_t launch_gemv_tc(const uint32_t* packed, const float* s, const DecodePlan& p, float* o, uint8_t* ws,
                           unsigned* status, cudaStream_t st);

// Prefill GEMM on tcgen05. `status` is the device status word.
cudaError_t launch_gemm(const uint32_t* packed, const float* s, int out, int K,
                        const uint16_t* u_bf16, int tokens, float* o, unsigned* status,
                        cudaStream_t st);

}  // namespace lq
