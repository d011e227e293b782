// Decode 1-bit GEMV, batch 1..16 (LiftQuant paper note, "Key designs" 4: after
// the small matmul T* a, the layer is a 1-bit x float matmul with W_q followed
// by diag(s)):
//
//   o[c][r] = s[r] * sum_k sigma[r][k] u[c][k],  sigma = +1 if the bit is set.
//
// CUDA-core design. A CTA of 8 warps owns 32 consecutive rows (4 per warp).
// The lifted activations are staged chunk by chunk in shared memory with one
// pad word per 32 floats, so that lane l reading element b of its own word
// hits bank (l + b) mod 32: conflict-free. Every lane streams whole sign words
// (coalesced 128-byte warp loads, four words in flight per row) and applies
// each sign by flipping the float's sign bit (one shift + one LOP3 per bit,
// shared by all batch columns), accumulating in fp32. Warp-shuffle reduction,
// then the per-row scale in the epilogue.
#include "lq_internal.h"

namespace lq {
namespace {

constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;
constexpr int kChunkFloats = 16384;  // per CTA: NB * chunk_k floats staged at once

template <int NB>
__global__ void __launch_bounds__(kWarps * 32) gemv_kernel(const uint32_t* __restrict__ packed,
                                                           const float* __restrict__ s, int out, int K,
                                                           const float* __restrict__ u,
                                                           float* __restrict__ o) {
    extern __shared__ float us[];  // [NB][chunk_k + chunk_k/32]
    constexpr int chunk_k = (kChunkFloats / NB) / 1024 * 1024;  // multiple of 32 words
    constexpr int pitch = chunk_k + chunk_k / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = blockIdx.x * kRowsPerCta + warp * kRowsPerWarp;
    const int kw = K >> 5;  // words per row

    float acc[kRowsPerWarp][NB];
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i)
#pragma unroll
        for (int c = 0; c < NB; ++c) acc[i][c] = 0.f;

    for (int k0 = 0; k0 < K; k0 += chunk_k) {
        const int nk = min(chunk_k, K - k0);  // multiple of 32
        __syncthreads();
        for (int c = 0; c < NB; ++c)
            for (int k = threadIdx.x; k < nk; k += blockDim.x)
                us[c * pitch + k + (k >> 5)] = __ldg(u + (long long)c * K + k0 + k);
        __syncthreads();

        const int nw = nk >> 5;
        for (int w = lane; w < nw; w += 32) {
            uint32_t nwd[kRowsPerWarp];
#pragma unroll
            for (int i = 0; i < kRowsPerWarp; ++i) {
                int r = row0 + i;
                nwd[i] = r < out ? ~__ldg(packed + (long long)r * kw + (k0 >> 5) + w) : 0u;
            }
            const float* ub = us + 33 * w;
#pragma unroll
            for (int b = 0; b < 32; ++b) {
                float uv[NB];
#pragma unroll
                for (int c = 0; c < NB; ++c) uv[c] = ub[c * pitch + b];
#pragma unroll
                for (int i = 0; i < kRowsPerWarp; ++i) {
                    uint32_t m = (nwd[i] << (31 - b)) & 0x80000000u;  // sign bit set where sigma = -1
#pragma unroll
                    for (int c = 0; c < NB; ++c) acc[i][c] += __uint_as_float(__float_as_uint(uv[c]) ^ m);
                }
            }
        }
    }

#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int r = row0 + i;
#pragma unroll
        for (int c = 0; c < NB; ++c) {
            float v = acc[i][c];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            acc[i][c] = v;
        }
        if (lane == 0 && r < out) {
            const float sr = __ldg(s + r);
#pragma unroll
            for (int c = 0; c < NB; ++c) o[(long long)c * out + r] = sr * acc[i][c];
        }
    }
}

template <int NB>
cudaError_t launch_nb(const uint32_t* packed, const float* s, int out, int K, const float* u,
                      float* o, cudaStream_t st) {
    constexpr int chunk_k = (kChunkFloats / NB) / 1024 * 1024;
    const size_t smem = sizeof(float) * (size_t)NB * (chunk_k + chunk_k / 32);
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemv_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    dim3 grid((out + kRowsPerCta - 1) / kRowsPerCta);
    gemv_kernel<NB><<<grid, kWarps * 32, smem, st>>>(packed, s, out, K, u, o);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(const uint32_t* packed, const float* s, int out, int K, const float* u,
                        int batch, float* o, cudaStream_t st) {
    switch (batch) {
#define LQ_NB(n) case n: return launch_nb<n>(packed, s, out, K, u, o, st);
        LQ_NB(1) LQ_NB(2) LQ_NB(3) LQ_NB(4) LQ_NB(5) LQ_NB(6) LQ_NB(7) LQ_NB(8)
        LQ_NB(9) LQ_NB(10) LQ_NB(11) LQ_NB(12) LQ_NB(13) LQ_NB(14) LQ_NB(15) LQ_NB(16)
#undef LQ_NB
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lq
