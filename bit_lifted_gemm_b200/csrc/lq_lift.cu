// Activation lift u = blockdiag(M^T) . T^{-1} . a (LiftQuant paper note,
// "Key designs" 3 and 4: the whitening inverse acts on the activations and the
// small matmul T* a = M T^{-1} a is computed once before the 1-bit matmul).
//
// Reading of the dimensions: T^{-1} is block diagonal (tblk x tblk blocks, or
// the identity); M^T is applied to each run of d consecutive whitened
// channels, block b producing lifted coordinates [b*D, (b+1)*D). Lifted
// entries past (in/d)*D up to K are zero.
//
// One CTA owns G consecutive d-blocks (channels [c0, c0 + G*d)) and a tile of
// tokens. It stages the activations of every whitening block that its channels
// touch in shared memory, forms a' = T^{-1} a for its own channels only (each
// row of T^{-1} is read by exactly one CTA per token tile), then lifts from
// shared memory. Two variants:
//   * decode (<= 16 tokens): one warp per channel reads its T^{-1} row with
//     coalesced loads and reduces the per-token dot products by shuffles; this
//     is HBM-bound on the T^{-1} bytes.
//   * prefill (32-token tiles): T^{-1} rows are staged in shared memory and each
//     thread forms 8 tokens x 1 channel with float4 broadcasts.
// Accumulation is fp32; bf16 output rounds to nearest even.
#include <cuda_bf16.h>

#include "lq_internal.h"

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

__device__ __forceinline__ float load_act(const void* a, int a_bf16, long long idx) {
    if (a_bf16) {
        unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(a) + idx);
        return __uint_as_float((unsigned)h << 16);
    }
    return __ldg(reinterpret_cast<const float*>(a) + idx);
}

__device__ __forceinline__ void store_u(void* u, int u_bf16, long long idx, float v) {
    if (u_bf16)
        reinterpret_cast<__nv_bfloat16*>(u)[idx] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float*>(u)[idx] = v;
}

// Channel range of this CTA and the span of input channels it must stage.
struct Range {
    int blk0, nblk, c0, C, lo, hi;
};

__device__ __forceinline__ Range cta_range(const LiftArgs& p) {
    Range r;
    r.blk0 = blockIdx.x * p.G;
    int nb = p.in / p.d - r.blk0;
    r.nblk = nb < p.G ? nb : p.G;
    r.c0 = r.blk0 * p.d;
    r.C = r.nblk * p.d;
    if (p.tinv) {
        r.lo = (r.c0 / p.tblk) * p.tblk;
        int hi = ((r.c0 + r.C - 1) / p.tblk + 1) * p.tblk;
        r.hi = hi < p.in ? hi : p.in;
    } else {
        r.lo = r.c0;
        r.hi = r.c0 + r.C;
    }
    return r;
}

// Lift from shared a' ([C][TB], tokens contiguous) and write u; the last CTA in x
// also zeroes the padded tail of the lifted axis.
template <int TB, int TT>
__device__ __forceinline__ void lift_and_store(const LiftArgs& p, const Range& r, const float* Ms,
                                               const float* aps, int t0, int nt) {
    const int nk = r.nblk * p.D;
    const int ngroups = (nt + TT - 1) / TT;
    for (int item = threadIdx.x; item < nk * ngroups; item += blockDim.x) {
        int kl = item % nk, tg = item / nk;
        int bl = kl / p.D, j = kl - bl * p.D;
        float acc[TT];
#pragma unroll
        for (int q = 0; q < TT; ++q) acc[q] = 0.f;
        for (int i = 0; i < p.d; ++i) {
            float m = Ms[i * p.D + j];
            const float* ar = aps + (bl * p.d + i) * TB + tg * TT;
#pragma unroll
            for (int q = 0; q < TT; ++q) acc[q] = fmaf(m, ar[q], acc[q]);
        }
        long long kk = (long long)r.blk0 * p.D + kl;
#pragma unroll
        for (int q = 0; q < TT; ++q) {
            int t = tg * TT + q;
            if (t < nt) store_u(p.u, p.u_bf16, (long long)(t0 + t) * p.K + kk, acc[q]);
        }
    }
    if (blockIdx.x == gridDim.x - 1) {
        const int kreal = (p.in / p.d) * p.D;
        const int npad = p.K - kreal;
        for (int item = threadIdx.x; item < npad * nt; item += blockDim.x) {
            int t = item / npad, k = kreal + item % npad;
            store_u(p.u, p.u_bf16, (long long)(t0 + t) * p.K + k, 0.f);
        }
    }
}

// ---------------------------------------------------------------- decode variant
constexpr int DEC_TB = 16;

__global__ void __launch_bounds__(256) lift_decode_kernel(LiftArgs p) {
    // A programmatically dependent consumer (the decode GEMV) may start now: it
    // streams its weights and waits for this grid before reading u.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ float smem[];
    const Range r = cta_range(p);
    const int t0 = blockIdx.y * DEC_TB;
    const int nt = min(DEC_TB, p.batch - t0);
    const int span = r.hi - r.lo;
    float* Ms = smem;                       // [d*D], padded to 16 bytes
    float* as = Ms + ((p.d * p.D + 3) & ~3); // [DEC_TB][span]: token-major, so lanes read consecutive channels
    float* aps = as + span * DEC_TB;        // [C][DEC_TB]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    // The T^{-1} rows dominate this kernel's HBM traffic: request each warp's
    // first two rows (up to 256 floats each) before anything else.
    const bool vec = p.tinv && (p.tblk & 3) == 0 && p.tblk <= 256;
    float4 tpre[2][2];
#pragma unroll
    for (int sl = 0; sl < 2; ++sl)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int ch = warp + sl * nwarps, j4 = lane + 32 * q;
            tpre[sl][q] = (vec && ch < r.C && j4 < (p.tblk >> 2))
                              ? __ldg(reinterpret_cast<const float4*>(p.tinv + (long long)(r.c0 + ch) * p.tblk) + j4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        }

    for (int i = threadIdx.x; i < p.d * p.D; i += blockDim.x) Ms[i] = __ldg(p.M + i);
    for (int i = threadIdx.x; i < span * nt; i += blockDim.x) {
        int t = i / span, j = i - t * span;
        as[t * span + j] = load_act(p.a, p.a_bf16, (long long)(t0 + t) * p.in + r.lo + j);
    }
    __syncthreads();

    if (vec) {
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
            const int ch = warp + sl * nwarps;
            if (ch >= r.C) continue;  // warp-uniform
            const int c = r.c0 + ch;
            const int base = (c / p.tblk) * p.tblk - r.lo;
            float acc[DEC_TB];
#pragma unroll
            for (int t = 0; t < DEC_TB; ++t) acc[t] = 0.f;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int j4 = lane + 32 * q;
                if (j4 < (p.tblk >> 2)) {
                    const float4 tv = tpre[sl][q];
                    const float* a0 = as + base + 4 * j4;  // span and base are multiples of 4 here
#pragma unroll
                    for (int t = 0; t < DEC_TB; ++t) {
                        if (t < nt) {
                            const float4 x = *reinterpret_cast<const float4*>(a0 + t * span);
                            float s = acc[t];
                            s = fmaf(tv.x, x.x, s);
                            s = fmaf(tv.y, x.y, s);
                            s = fmaf(tv.z, x.z, s);
                            s = fmaf(tv.w, x.w, s);
                            acc[t] = s;
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < DEC_TB; ++t) {
                if (t < nt) {
                    float v = acc[t];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    if (lane == 0) aps[ch * DEC_TB + t] = v;
                }
            }
        }
    }
    if (p.tinv) {
        // channels beyond the two preloaded per warp, or whitening blocks that are
        // not float4-friendly
        for (int ch = vec ? warp + 2 * nwarps : warp; ch < r.C; ch += nwarps) {
            const int c = r.c0 + ch;
            const int base = (c / p.tblk) * p.tblk - r.lo;
            const float* row = p.tinv + (long long)c * p.tblk;  // row (c mod tblk) of block c/tblk
            float acc[DEC_TB];
#pragma unroll
            for (int t = 0; t < DEC_TB; ++t) acc[t] = 0.f;
            if ((p.tblk & 3) == 0) {
                for (int j4 = lane; j4 < (p.tblk >> 2); j4 += 32) {
                    float4 tv = __ldg(reinterpret_cast<const float4*>(row) + j4);
                    const float* a0 = as + base + 4 * j4;
#pragma unroll
                    for (int t = 0; t < DEC_TB; ++t) {
                        if (t < nt) {
                            const float4 x = *reinterpret_cast<const float4*>(a0 + t * span);
                            float s = acc[t];
                            s = fmaf(tv.x, x.x, s);
                            s = fmaf(tv.y, x.y, s);
                            s = fmaf(tv.z, x.z, s);
                            s = fmaf(tv.w, x.w, s);
                            acc[t] = s;
                        }
                    }
                }
            } else {
                for (int j = lane; j < p.tblk; j += 32) {
                    float tv = __ldg(row + j);
#pragma unroll
                    for (int t = 0; t < DEC_TB; ++t)
                        if (t < nt) acc[t] = fmaf(tv, as[t * span + base + j], acc[t]);
                }
            }
#pragma unroll
            for (int t = 0; t < DEC_TB; ++t) {
                if (t < nt) {
                    float v = acc[t];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    if (lane == 0) aps[ch * DEC_TB + t] = v;
                }
            }
        }
    } else {
        for (int i = threadIdx.x; i < r.C * nt; i += blockDim.x) {
            int ch = i / nt, t = i - ch * nt;
            aps[ch * DEC_TB + t] = as[t * span + ch];  // span = C, lo = c0 without whitening
        }
    }
    __syncthreads();
    lift_and_store<DEC_TB, 1>(p, r, Ms, aps, t0, nt);
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

__device__ __forceinline__ float4 load_act4(const void* a, int a_bf16, long long idx) {
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

template <int Q, int NTOK>
__global__ void __launch_bounds__(64) lift_warp_kernel(LiftArgs p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // see lift_decode_kernel
    const int lane = threadIdx.x & 31;
    const int blk = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int nblocks = p.in / p.d;
    if (blk >= nblocks) return;  // whole warp
    const int c0 = blk * p.d;
    const int tb4 = p.tblk >> 2;
    float4 Tv[WARP_MAXD][Q > 0 ? Q : 1];
#pragma unroll
    for (int i = 0; i < WARP_MAXD; ++i)
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            const int j4 = lane + 32 * q;
            Tv[i][q] = i < p.d && j4 < tb4
                           ? __ldg(reinterpret_cast<const float4*>(p.tinv + (long long)(c0 + i) * p.tblk) + j4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    float mc[2][WARP_MAXD];  // M[i][lane], M[i][lane + 32]
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < WARP_MAXD; ++i) {
            const int j = lane + 32 * h;
            mc[h][i] = i < p.d && j < p.D ? __ldg(p.M + i * p.D + j) : 0.f;
        }
    const int ba = Q > 0 ? (c0 / p.tblk) * p.tblk : 0;            // whitening block of the first channel
    const int bb = Q > 0 ? ((c0 + p.d - 1) / p.tblk) * p.tblk : 0;  // ... and of the last (ba or the next one)
    for (int tb = 0; tb < p.batch; tb += NTOK) {
        // the activation slices of NTOK tokens are requested before any is used
        float4 A0[NTOK][Q > 0 ? Q : 1], A1[NTOK][Q > 0 ? Q : 1];
        float ap[NTOK][WARP_MAXD];
#pragma unroll
        for (int n = 0; n < NTOK; ++n) {
            const int t = tb + n;
            const long long arow = (long long)t * p.in;
            if (Q > 0) {
#pragma unroll
                for (int q = 0; q < Q; ++q) {
                    const int j4 = lane + 32 * q;
                    const bool ok = t < p.batch && j4 < tb4;
                    A0[n][q] = ok ? load_act4(p.a, p.a_bf16, arow + ba + 4 * j4) : make_float4(0.f, 0.f, 0.f, 0.f);
                    A1[n][q] = ok && bb != ba ? load_act4(p.a, p.a_bf16, arow + bb + 4 * j4) : A0[n][q];
                }
            } else {
#pragma unroll
                for (int i = 0; i < WARP_MAXD; ++i)
                    ap[n][i] = t < p.batch && i < p.d ? load_act(p.a, p.a_bf16, arow + c0 + i) : 0.f;
            }
        }
        if (Q > 0) {
#pragma unroll
            for (int n = 0; n < NTOK; ++n)
#pragma unroll
                for (int i = 0; i < WARP_MAXD; ++i) {
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
                    for (int i = 0; i < WARP_MAXD; ++i) acc = fmaf(mc[h][i], ap[n][i], acc);
                    store_u(p.u, p.u_bf16, (long long)t * p.K + (long long)blk * p.D + j, acc);
                }
            }
        }
    }
    if (blk == nblocks - 1) {  // zero the padded tail of the lifted axis
        const int kreal = nblocks * p.D;
        for (int t = 0; t < p.batch; ++t)
            for (int k = kreal + lane; k < p.K; k += 32) store_u(p.u, p.u_bf16, (long long)t * p.K + k, 0.f);
    }
}

// ---------------------------------------------------------------- prefill variant
constexpr int PRE_TB = 32;  // tokens per CTA
constexpr int PRE_TT = 8;   // tokens per thread

__global__ void __launch_bounds__(256) lift_prefill_kernel(LiftArgs p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // see lift_decode_kernel
    extern __shared__ float smem[];
    const Range r = cta_range(p);
    const int t0 = blockIdx.y * PRE_TB;
    const int nt = min(PRE_TB, p.batch - t0);
    const int span = r.hi - r.lo;
    const int tstride = p.tblk + 1;             // padded T^{-1} row pitch in shared memory
    float* Ms = smem;                           // [d*D], padded to 16 bytes
    float* as = Ms + ((p.d * p.D + 3) & ~3);    // [span][PRE_TB]
    float* aps = as + span * PRE_TB;            // [C][PRE_TB]
    float* Ts = aps + r.C * PRE_TB;             // [C][tblk+1] (only with tinv)

    for (int i = threadIdx.x; i < p.d * p.D; i += blockDim.x) Ms[i] = __ldg(p.M + i);
    for (int i = threadIdx.x; i < span * PRE_TB; i += blockDim.x) {
        int t = i / span, j = i - t * span;
        as[j * PRE_TB + t] = t < nt ? load_act(p.a, p.a_bf16, (long long)(t0 + t) * p.in + r.lo + j) : 0.f;
    }
    if (p.tinv) {
        for (int i = threadIdx.x; i < r.C * p.tblk; i += blockDim.x) {
            int ch = i / p.tblk, j = i - ch * p.tblk;
            Ts[ch * tstride + j] = __ldg(p.tinv + (long long)(r.c0 + ch) * p.tblk + j);
        }
    }
    __syncthreads();

    if (p.tinv) {
        constexpr int NG = PRE_TB / PRE_TT;
        for (int item = threadIdx.x; item < r.C * NG; item += blockDim.x) {
            int ch = item / NG, tg = item - ch * NG;
            int c = r.c0 + ch;
            const float* trow = Ts + ch * tstride;
            const float* acol = as + ((c / p.tblk) * p.tblk - r.lo) * PRE_TB + tg * PRE_TT;
            float acc[PRE_TT];
#pragma unroll
            for (int q = 0; q < PRE_TT; ++q) acc[q] = 0.f;
            for (int j = 0; j < p.tblk; ++j) {
                float tv = trow[j];
                float4 x0 = *reinterpret_cast<const float4*>(acol + j * PRE_TB);
                float4 x1 = *reinterpret_cast<const float4*>(acol + j * PRE_TB + 4);
                acc[0] = fmaf(tv, x0.x, acc[0]); acc[1] = fmaf(tv, x0.y, acc[1]);
                acc[2] = fmaf(tv, x0.z, acc[2]); acc[3] = fmaf(tv, x0.w, acc[3]);
                acc[4] = fmaf(tv, x1.x, acc[4]); acc[5] = fmaf(tv, x1.y, acc[5]);
                acc[6] = fmaf(tv, x1.z, acc[6]); acc[7] = fmaf(tv, x1.w, acc[7]);
            }
            float* dst = aps + ch * PRE_TB + tg * PRE_TT;
            *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
    } else {
        for (int i = threadIdx.x; i < r.C * PRE_TB; i += blockDim.x) aps[i] = as[i];
    }
    __syncthreads();
    lift_and_store<PRE_TB, PRE_TT>(p, r, Ms, aps, t0, nt);
}

// Raise a kernel's dynamic shared-memory limit once per device to the largest
// size requested so far (cudaFuncSetAttribute is not a stream operation, so
// repeated calls are avoided on launch paths that may be graph-captured).
cudaError_t raise_smem_limit(const void* fn, size_t bytes, int which) {
    static size_t granted[2][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && granted[which][dev] >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev < 64) granted[which][dev] = bytes;
    return e;
}

}  // namespace

cudaError_t launch_lift(const void* a, bool a_bf16, int batch, int in, const float* tinv, int tblk,
                        const float* M, int d, int D, void* u, bool u_bf16, int K, cudaStream_t st) {
    LiftArgs p;
    p.a = a; p.tinv = tinv; p.M = M; p.u = u;
    p.a_bf16 = a_bf16; p.u_bf16 = u_bf16;
    p.batch = batch; p.in = in; p.tblk = tinv ? tblk : 1; p.d = d; p.D = D; p.K = K;
    const int nblocks = in / d;
    const bool decode = batch <= DEC_TB;
    // one warp per d-block for the smallest batches (up to 4 tokens, 2 with
    // 256-wide whitening blocks), the shared-memory kernels otherwise
    const bool warp_ok = d <= WARP_MAXD && D <= WARP_MAXDD &&
                         (!tinv || (tblk % 4 == 0 && tblk >= d && tblk <= 256)) &&
                         (batch <= 2 || (batch <= 4 && (!tinv || tblk <= 128)));
    if (warp_ok) {
        const dim3 grid((in / d + 1) / 2);
        const int q = !tinv ? 0 : tblk <= 128 ? 1 : 2;
        if (batch == 1) {
            if (q == 0) lift_warp_kernel<0, 1><<<grid, 64, 0, st>>>(p);
            else if (q == 1) lift_warp_kernel<1, 1><<<grid, 64, 0, st>>>(p);
            else lift_warp_kernel<2, 1><<<grid, 64, 0, st>>>(p);
        } else if (batch == 2) {
            if (q == 0) lift_warp_kernel<0, 2><<<grid, 64, 0, st>>>(p);
            else if (q == 1) lift_warp_kernel<1, 2><<<grid, 64, 0, st>>>(p);
            else lift_warp_kernel<2, 2><<<grid, 64, 0, st>>>(p);
        } else {
            if (q == 0) lift_warp_kernel<0, 4><<<grid, 64, 0, st>>>(p);
            else lift_warp_kernel<1, 4><<<grid, 64, 0, st>>>(p);
        }
        return cudaGetLastError();
    }
    // channels per CTA: ~16 for decode (many CTAs to stream T^{-1}), ~64 for prefill
    int G = (decode ? 16 : 64) / d;
    if (G < 1) G = 1;
    if (G > nblocks) G = nblocks;
    p.G = G;
    const int C = G * d;
    // widest staged span: the whitening blocks that C consecutive channels can touch
    int span = tinv ? ((C + tblk - 2) / tblk + 1) * tblk : C;
    if (span > in) span = in;
    const size_t mpad = (size_t)((d * D + 3) & ~3);
    dim3 grid((nblocks + G - 1) / G, 1);
    size_t smem;
    if (decode) {
        grid.y = (batch + DEC_TB - 1) / DEC_TB;
        smem = sizeof(float) * (mpad + (size_t)span * DEC_TB + (size_t)C * DEC_TB);
        if (smem > 48 * 1024) {
            cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(lift_decode_kernel), smem, 0);
            if (e != cudaSuccess) return e;
        }
        lift_decode_kernel<<<grid, 256, smem, st>>>(p);
    } else {
        grid.y = (batch + PRE_TB - 1) / PRE_TB;
        smem = sizeof(float) * (mpad + (size_t)span * PRE_TB + (size_t)C * PRE_TB +
                                (tinv ? (size_t)C * (tblk + 1) : 0));
        if (smem > 48 * 1024) {
            cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(lift_prefill_kernel), smem, 1);
            if (e != cudaSuccess) return e;
        }
        lift_prefill_kernel<<<grid, 256, smem, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace lq
