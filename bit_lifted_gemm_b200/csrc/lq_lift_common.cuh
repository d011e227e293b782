// Pieces of the activation lift shared by the block-whitening lift kernels
// (lq_lift.cu) and the CUDA-core Kronecker lift (lq_lift_kron.cu): the argument
// block, activation / output accessors (bounds-checked in the debug build) and
// the one-warp-per-d-block lift (LiftQuant paper note, "Key designs" 3 and 4).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "lq_debug.cuh"

namespace lq {
namespace {

struct LiftArgs {
    const void* a;
    const float* tinv;
    const float* M;
    void* u;
    int a_bf16, u_bf16;
    int batch, in, tblk, d, D, K;
    int G;   // d-blocks per CTA
};

// Element idx of an activation buffer of n elements (n bounds the debug build's check).
__device__ __forceinline__ float load_act(const void* a, int a_bf16, long long idx, long long n) {
    if (!LQ_IN_BOUNDS(idx, n)) return 0.f;
    if (a_bf16) {
        unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(a) + idx);
        return __uint_as_float((unsigned)h << 16);
    }
    return __ldg(reinterpret_cast<const float*>(a) + idx);
}

// Element idx of u, a buffer of n elements (n bounds the debug build's check).
__device__ __forceinline__ void store_u(void* u, int u_bf16, long long idx, long long n, float v) {
    if (!LQ_IN_BOUNDS(idx, n)) return;
    if (u_bf16)
        reinterpret_cast<__nv_bfloat16*>(u)[idx] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float*>(u)[idx] = v;
}

// ------------------------------------------------ decode variant: one warp per d-block
// For decode batches with small blocks (d <= 16, D <= 64, tblk >= d): warp w
// owns d-block w. It issues all its loads at once -- the d rows of T^{-1} (Q
// float4 per lane; Q = 0 means T = identity), its column(s) of M, the activation
// slices of NTOK tokens -- then forms each a'[i] with a butterfly reduction
// (every lane ends with all d values) and lifts in registers: lane j writes
// u[blk*D + j]. No shared memory, no block barrier: one dependent round trip to
// memory per NTOK tokens.
constexpr int WARP_MAXD = 16;
constexpr int WARP_MAXDD = 64;

// Elements idx .. idx + 3 of an activation buffer of n elements.
__device__ __forceinline__ float4 load_act4(const void* a, int a_bf16, long long idx, long long n) {
    if (!LQ_IN_BOUNDS(idx + 3, n)) return make_float4(0.f, 0.f, 0.f, 0.f);
    if (a_bf16) {
        const uint2 h = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const unsigned short*>(a) + idx));
        return make_float4(__uint_as_float(h.x << 16), __uint_as_float(h.x & 0xffff0000u),
                           __uint_as_float(h.y << 16), __uint_as_float(h.y & 0xffff0000u));
    }
    return __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a) + idx));
}

__device__ __forceinline__ float dot4(const float4& x, const float4& y, float s) {
    s = fmaf(x.x, y.x, s);
    s = fmaf(x.y, y.y, s);
    s = fmaf(x.z, y.z, s);
    return fmaf(x.w, y.w, s);
}

// d-block blk of the lift, computed by one warp (lane = lane index); see above.
// MAXD >= d bounds the registers held per warp (the rows of T^-1, M and a').
template <int Q, int NTOK, int MAXD>
__device__ __forceinline__ void lift_block(const LiftArgs& p, int blk, int lane) {
    const int nblocks = p.in / p.d;
    const int c0 = blk * p.d;
    const int tb4 = p.tblk >> 2;
    float4 Tv[MAXD][Q > 0 ? Q : 1];
#pragma unroll
    for (int i = 0; i < MAXD; ++i)
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            const int j4 = lane + 32 * q;
            Tv[i][q] = i < p.d && j4 < tb4
                           ? __ldg(reinterpret_cast<const float4*>(p.tinv + (long long)(c0 + i) * p.tblk) + j4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    float mc[2][MAXD];  // M[i][lane], M[i][lane + 32]
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < MAXD; ++i) {
            const int j = lane + 32 * h;
            mc[h][i] = i < p.d && j < p.D ? __ldg(p.M + i * p.D + j) : 0.f;
        }
    // T^-1 and M do not depend on the kernel before this one; the activations
    // (and the u it may still read) do: wait for it here when launched as a
    // programmatic dependent (a no-op otherwise)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int ba = Q > 0 ? (c0 / p.tblk) * p.tblk : 0;            // whitening block of the first channel
    const int bb = Q > 0 ? ((c0 + p.d - 1) / p.tblk) * p.tblk : 0;  // ... and of the last (ba or the next one)
    for (int tb = 0; tb < p.batch; tb += NTOK) {
        // the activation slices of NTOK tokens are requested before any is used
        float4 A0[NTOK][Q > 0 ? Q : 1], A1[NTOK][Q > 0 ? Q : 1];
        float ap[NTOK][MAXD];
#pragma unroll
        for (int n = 0; n < NTOK; ++n) {
            const int t = tb + n;
            const long long arow = (long long)t * p.in;
            if (Q > 0) {
#pragma unroll
                for (int q = 0; q < Q; ++q) {
                    const int j4 = lane + 32 * q;
                    const bool ok = t < p.batch && j4 < tb4;
                    A0[n][q] = ok ? load_act4(p.a, p.a_bf16, arow + ba + 4 * j4, (long long)p.batch * p.in) : make_float4(0.f, 0.f, 0.f, 0.f);
                    A1[n][q] = ok && bb != ba ? load_act4(p.a, p.a_bf16, arow + bb + 4 * j4, (long long)p.batch * p.in) : A0[n][q];
                }
            } else {
#pragma unroll
                for (int i = 0; i < MAXD; ++i)
                    ap[n][i] = t < p.batch && i < p.d ? load_act(p.a, p.a_bf16, arow + c0 + i, (long long)p.batch * p.in) : 0.f;
            }
        }
        if (Q > 0) {
#pragma unroll
            for (int n = 0; n < NTOK; ++n)
#pragma unroll
                for (int i = 0; i < MAXD; ++i) {
                    ap[n][i] = 0.f;
                    if (i < p.d) {
                        const bool second = c0 + i >= bb;
                        float sum = 0.f;
#pragma unroll
                        for (int q = 0; q < Q; ++q) sum = dot4(Tv[i][q], second ? A1[n][q] : A0[n][q], sum);
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                        ap[n][i] = sum;
                    }
                }
        }
#pragma unroll
        for (int n = 0; n < NTOK; ++n) {
            const int t = tb + n;
            if (t >= p.batch) break;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h;
                if (j < p.D) {
                    float acc = 0.f;
#pragma unroll
                    for (int i = 0; i < MAXD; ++i) acc = fmaf(mc[h][i], ap[n][i], acc);
                    store_u(p.u, p.u_bf16, (long long)t * p.K + (long long)blk * p.D + j, (long long)p.batch * p.K, acc);
                }
            }
        }
    }
    if (blk == nblocks - 1) {  // zero the padded tail of the lifted axis
        const int kreal = nblocks * p.D;
        for (int t = 0; t < p.batch; ++t)
            for (int k = kreal + lane; k < p.K; k += 32) store_u(p.u, p.u_bf16, (long long)t * p.K + k, (long long)p.batch * p.K, 0.f);
    }
}


}  // namespace
}  // namespace lq
