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

#include <algorithm>

#include "lq_internal.h"
#include "lq_lift_common.cuh"

namespace lq {
namespace {

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
            if (t < nt) store_u(p.u, p.u_bf16, (long long)(t0 + t) * p.K + kk, (long long)p.batch * p.K, acc[q]);
        }
    }
    if (blockIdx.x == gridDim.x - 1) {
        const int kreal = (p.in / p.d) * p.D;
        const int npad = p.K - kreal;
        for (int item = threadIdx.x; item < npad * nt; item += blockDim.x) {
            int t = item / npad, k = kreal + item % npad;
            store_u(p.u, p.u_bf16, (long long)(t0 + t) * p.K + k, (long long)p.batch * p.K, 0.f);
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
        as[t * span + j] = load_act(p.a, p.a_bf16, (long long)(t0 + t) * p.in + r.lo + j, (long long)p.batch * p.in);
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

template <int Q, int NTOK, int MAXD>
__global__ void __launch_bounds__(64) lift_warp_kernel(LiftArgs p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // see lift_decode_kernel
    const int blk = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (blk >= p.in / p.d) return;  // whole warp
    lift_block<Q, NTOK, MAXD>(p, blk, threadIdx.x & 31);
}

// Few registers per warp let a GEMV CTA become resident beside the lift's CTAs
// (and start its prologue) while the lift runs. The lift is itself launched as
// a programmatic dependent of the kernel before it: its CTAs may start (and
// stream T^-1) while that kernel finishes, and wait for it before reading the
// activations.
template <int Q, int NTOK>
void launch_warp_lift(const LiftArgs& p, int d, dim3 grid, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(64, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (d <= 8)
        cudaLaunchKernelEx(&cfg, lift_warp_kernel<Q, NTOK, 8>, p);
    else if (d <= 12)
        cudaLaunchKernelEx(&cfg, lift_warp_kernel<Q, NTOK, 12>, p);
    else
        cudaLaunchKernelEx(&cfg, lift_warp_kernel<Q, NTOK, 16>, p);
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
        as[j * PRE_TB + t] = t < nt ? load_act(p.a, p.a_bf16, (long long)(t0 + t) * p.in + r.lo + j, (long long)p.batch * p.in) : 0.f;
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

// ------------------------------------------------ prefill variant, register tiled
// For whitening blocks of 16..128 channels (tblk % 8 == 0): a CTA owns G
// consecutive d-blocks (C <= min(120, tblk) channels, so they touch at most two
// whitening blocks) and 64 tokens. T^-1 rows and the activations of both
// whitening blocks are staged transposed in shared memory; each thread forms
// a' for 4 channels x 8 tokens (32 accumulators, three 16-byte shared loads per
// 32 FMAs), then the lift reads a' from shared memory. A channel group of 4
// never straddles whitening blocks: each block's channels are padded to a
// multiple of 4.
constexpr int P2_TT = 64;              // tokens per CTA
constexpr int P2_AP = 76;              // pitch (floats) of a row of 64 staged tokens (see p2_pos)
constexpr int P2_TP = 132;             // pitch (floats) of a staged T^-1 column (<= 128 padded channels)
constexpr int P2_CMAX = 120;           // channels per CTA
constexpr int P2_JC = 64;              // whitening-block columns staged at a time

// Position of token t in a staged row: token group g = t/8 keeps its first four
// tokens at 4g and its last four at 36 + 4g, so the eight 16-byte chunks that
// the eight token groups of a quarter-warp read fall in distinct bank groups.
__device__ __forceinline__ int p2_pos(int t) { return ((t >> 2) & 1) * 36 + (t >> 3) * 4 + (t & 3); }

__host__ __device__ inline size_t prefill2_smem(int tblk, int d, int D) {
    const size_t jc = tblk < P2_JC ? tblk : P2_JC;
    return sizeof(float) * ((size_t)2 * jc * P2_AP + (size_t)jc * P2_TP + (((size_t)d * D + 3) & ~(size_t)3));
}

__global__ void __launch_bounds__(256) lift_prefill2_kernel(LiftArgs p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // see lift_decode_kernel
    extern __shared__ __align__(16) float smem[];
    const int nblocks = p.in / p.d;
    const int b0 = blockIdx.x * p.G, b1 = min(nblocks, b0 + p.G);
    const int c0 = b0 * p.d, C = (b1 - b0) * p.d;
    const int t0 = blockIdx.y * P2_TT, nt = min(P2_TT, p.batch - t0);
    const int kb0 = c0 / p.tblk;                          // first whitening block touched
    const int split = min(C, (kb0 + 1) * p.tblk - c0);    // channels [0, split) lie in block kb0
    const int PA = (split + 3) & ~3, PB = (C - split + 3) & ~3;
    const int nbl = split < C ? 2 : 1;
    const int JC = min(P2_JC, p.tblk);                 // columns j staged per pass
    float* as = smem;                                   // [2][JC][P2_AP]: a[t][block bl, j0 + j]
    float* Ts = as + 2 * JC * P2_AP;                   // [JC][P2_TP]: T^-1[c][j0 + j] at [j][padded c]
    float* Ms = Ts + JC * P2_TP;                       // [d*D]
    float* aps = as;                                    // [C][P2_AP]: a' (reuses the activation area)

    for (int i = threadIdx.x; i < p.d * p.D; i += blockDim.x) Ms[i] = __ldg(p.M + i);
    // a' for 4 padded channels x 8 tokens per thread; a warp holds 4 channel
    // groups x 8 token groups (broadcast-friendly shared loads)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cg = warp * 4 + (lane >> 3), tg = lane & 7;
    const int pc0 = 4 * cg;
    const bool active = pc0 < PA + PB;
    const int bl = pc0 < PA ? 0 : 1;
    float acc[4][8];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int t = 0; t < 8; ++t) acc[q][t] = 0.f;
    for (int j0 = 0; j0 < p.tblk; j0 += JC) {
        const int jc = min(JC, p.tblk - j0);  // a multiple of 8
        if (j0) __syncthreads();  // the previous columns have been consumed
        // Activations: chunk = 8 consecutive channels of one token (one 16-byte load
        // of bf16, two of fp32); lanes run over tokens, so the transposed stores
        // are conflict-free. Eight chunks per thread are requested before any store.
        {
            const int jgs = jc >> 3;                         // chunks per whitening block and token
            const int nchunk = nbl * jgs * P2_TT;
            for (int base = threadIdx.x; base < nchunk; base += 8 * 256) {
                float v[8][8];
#pragma unroll
                for (int u8 = 0; u8 < 8; ++u8) {
                    const int i = base + u8 * 256, t = i % P2_TT, r = i / P2_TT;
                    const int jg = r % jgs, bl2 = r / jgs;
                    const long long idx = (long long)(t0 + t) * p.in + (kb0 + bl2) * p.tblk + j0 + 8 * jg;
                    if (i < nchunk && t < nt) {
                        if (p.a_bf16) {
                            const uint4 h = __ldg(reinterpret_cast<const uint4*>(
                                reinterpret_cast<const unsigned short*>(p.a) + idx));
                            const uint32_t w[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                v[u8][2 * q] = __uint_as_float(w[q] << 16);
                                v[u8][2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
                            }
                        } else {
                            const float4 f0 = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.a) + idx));
                            const float4 f1 =
                                __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.a) + idx) + 1);
                            v[u8][0] = f0.x; v[u8][1] = f0.y; v[u8][2] = f0.z; v[u8][3] = f0.w;
                            v[u8][4] = f1.x; v[u8][5] = f1.y; v[u8][6] = f1.z; v[u8][7] = f1.w;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 8; ++q) v[u8][q] = 0.f;
                    }
                }
#pragma unroll
                for (int u8 = 0; u8 < 8; ++u8) {
                    const int i = base + u8 * 256, t = i % P2_TT, r = i / P2_TT;
                    const int jg = r % jgs, bl2 = r / jgs;
                    if (i < nchunk) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) as[(bl2 * JC + 8 * jg + q) * P2_AP + p2_pos(t)] = v[u8][q];
                    }
                }
            }
        }
        // T^-1 rows: chunk = 4 consecutive j of one padded channel (one 16-byte
        // load); lanes run over channels, so the transposed stores are conflict-free.
        {
            const int j4s = jc >> 2;
            const int nchunk = 128 * j4s;                    // padded channels 0..127 (those >= PA + PB are zero)
            for (int base = threadIdx.x; base < nchunk; base += 8 * 256) {
                float4 v[8];
#pragma unroll
                for (int u8 = 0; u8 < 8; ++u8) {
                    const int i = base + u8 * 256, pc = i & 127, j4 = i >> 7;
                    const int lc = pc < PA ? pc : split + (pc - PA);
                    const bool valid = i < nchunk && (pc < PA ? pc < split : pc < PA + PB && lc < C);
                    v[u8] = valid ? __ldg(reinterpret_cast<const float4*>(p.tinv + (long long)(c0 + lc) * p.tblk + j0) + j4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u8 = 0; u8 < 8; ++u8) {
                    const int i = base + u8 * 256, pc = i & 127, j4 = i >> 7;
                    if (i < nchunk) {
                        float* dst = Ts + 4 * j4 * P2_TP + pc;
                        dst[0] = v[u8].x;
                        dst[P2_TP] = v[u8].y;
                        dst[2 * P2_TP] = v[u8].z;
                        dst[3 * P2_TP] = v[u8].w;
                    }
                }
            }
        }
        __syncthreads();
        if (active) {
            const float* ab = as + bl * JC * P2_AP + 4 * tg;
            const float* tb = Ts + pc0;
#pragma unroll 4
            for (int j = 0; j < jc; ++j) {
                const float4 x0 = *reinterpret_cast<const float4*>(ab + j * P2_AP);
                const float4 x1 = *reinterpret_cast<const float4*>(ab + j * P2_AP + 36);
                const float4 w = *reinterpret_cast<const float4*>(tb + j * P2_TP);
                const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                const float ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int t = 0; t < 8; ++t) acc[q][t] = fmaf(ws[q], xs[t], acc[q][t]);
            }
        }
    }
    __syncthreads();  // the activation area becomes a'
    if (active) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int pc = pc0 + q;
            const int lc = pc < PA ? pc : split + (pc - PA);
            if ((pc < PA ? pc < split : lc < C)) {
                float* dst = aps + lc * P2_AP + 4 * tg;
                *reinterpret_cast<float4*>(dst) = make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
                *reinterpret_cast<float4*>(dst + 36) = make_float4(acc[q][4], acc[q][5], acc[q][6], acc[q][7]);
            }
        }
    }
    __syncthreads();

    // lift: item = (lifted coordinate k of this CTA, token group of 8)
    const int nk = (b1 - b0) * p.D;
    for (int item = threadIdx.x; item < nk * (P2_TT / 8); item += blockDim.x) {
        const int kl = item % nk, g8 = item / nk;
        const int bl2 = kl / p.D, jj = kl - bl2 * p.D;
        float o[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) o[t] = 0.f;
        for (int i = 0; i < p.d; ++i) {
            const float m = Ms[i * p.D + jj];
            const float* ar = aps + (bl2 * p.d + i) * P2_AP + 4 * g8;
            const float4 x0 = *reinterpret_cast<const float4*>(ar);
            const float4 x1 = *reinterpret_cast<const float4*>(ar + 36);
            o[0] = fmaf(m, x0.x, o[0]); o[1] = fmaf(m, x0.y, o[1]); o[2] = fmaf(m, x0.z, o[2]); o[3] = fmaf(m, x0.w, o[3]);
            o[4] = fmaf(m, x1.x, o[4]); o[5] = fmaf(m, x1.y, o[5]); o[6] = fmaf(m, x1.z, o[6]); o[7] = fmaf(m, x1.w, o[7]);
        }
        const long long kk = (long long)b0 * p.D + kl;
#pragma unroll
        for (int t = 0; t < 8; ++t)
            if (8 * g8 + t < nt) store_u(p.u, p.u_bf16, (long long)(t0 + 8 * g8 + t) * p.K + kk, (long long)p.batch * p.K, o[t]);
    }
    if (blockIdx.x == gridDim.x - 1) {  // zero the padded tail of the lifted axis
        const int kreal = nblocks * p.D, npad = p.K - kreal;
        for (int i = threadIdx.x; i < npad * nt; i += blockDim.x)
            store_u(p.u, p.u_bf16, (long long)(t0 + i / npad) * p.K + kreal + i % npad, (long long)p.batch * p.K, 0.f);
    }
}

// Raise a kernel's dynamic shared-memory limit once per device to the largest
// size requested so far (cudaFuncSetAttribute is not a stream operation, so
// repeated calls are avoided on launch paths that may be graph-captured).
cudaError_t raise_smem_limit(const void* fn, size_t bytes, int which) {
    static size_t granted[3][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && granted[which][dev] >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev < 64) granted[which][dev] = bytes;
    return e;
}

}  // namespace

cudaError_t launch_lift(const void* a, bool a_bf16, int batch, int in, const float* tinv, int tblk,
                        const float* M, int d, int D, void* u, bool u_bf16, int K, unsigned* status,
                        cudaStream_t st) {
    if (lift_tc_supported(a_bf16, batch, in, tinv, tblk, d, D))
        return launch_lift_tc(static_cast<const uint16_t*>(a), batch, in, tinv, M, d, D, u, u_bf16, K, status, st);
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
            if (q == 0) launch_warp_lift<0, 1>(p, d, grid, st);
            else if (q == 1) launch_warp_lift<1, 1>(p, d, grid, st);
            else launch_warp_lift<2, 1>(p, d, grid, st);
        } else if (batch == 2) {
            if (q == 0) launch_warp_lift<0, 2>(p, d, grid, st);
            else if (q == 1) launch_warp_lift<1, 2>(p, d, grid, st);
            else launch_warp_lift<2, 2>(p, d, grid, st);
        } else {
            if (q == 0) launch_warp_lift<0, 4>(p, d, grid, st);
            else launch_warp_lift<1, 4>(p, d, grid, st);
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
    } else if (tinv && tblk % 8 == 0 && tblk >= 16 && tblk <= 128 && d <= P2_CMAX && d <= tblk &&
               prefill2_smem(tblk, d, D) <= 227 * 1024) {
        LiftArgs q = p;
        q.G = std::max(1, std::min(P2_CMAX, tblk) / d);
        const dim3 g2((nblocks + q.G - 1) / q.G, (batch + P2_TT - 1) / P2_TT);
        const size_t sm2 = prefill2_smem(tblk, d, D);
        cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(lift_prefill2_kernel), sm2, 2);
        if (e != cudaSuccess) return e;
        lift_prefill2_kernel<<<g2, 256, sm2, st>>>(q);
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

LQ_DEBUG_FLAG_TAKE(debug_take_lift)
