// Activation lift with a Kronecker-factored whitening (LiftQuant paper note,
// "Key designs" 3: T = diag(s1) (P1 kron P2) diag(s2), s2 constant over each
// d-block, so T^{-1} = diag(r2) (Q1 kron Q2) diag(r1) with r = 1/s, Q = P^{-1};
// the caller hands over the factors of T^{-1}). After the whitening comes the
// per-block lift u_blk = M^T a'_blk ("Key designs" 4).
//
// With in = n1 * n2 and one token's activations read as the n1 x n2 matrix X
// (row-major: element i1 * n2 + i2), (Q1 kron Q2) x is Q1 X Q2^T: in * (n1 + n2)
// multiply-adds instead of in^2, and (n1^2 + n2^2) floats of factors.
//
// The product is taken as Y = (Q1 X) Q2^T. A CTA that owns rows [c R, (c+1) R)
// of the result needs only its R rows of Q1 and the whole X of its token -- which
// it reads from global memory -- so a token can be spread over C CTAs with no
// exchange between them:
//   1. W = Q1[own rows] (r1 o X)      (R x n2, contraction over n1)
//   2. Y = W Q2^T                     (R x n2, contraction over n2)
//   3. a' = r2 o Y and the lift of the d-blocks inside its rows (C is chosen so
//      that R * n2 is a multiple of d: no block straddles two CTAs).
// Decode batches (<= 32 tokens) use up to 16 CTAs per token; larger batches keep
// whole tokens in one CTA, NT per CTA, in persistent CTAs that keep the factors
// in shared memory across token groups. All arithmetic is fp32 (fp32
// accumulation of n1 and then n2 products).
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "lq_internal.h"
#include "lq_lift_common.cuh"

namespace lq {
namespace {

constexpr int KR_THREADS = 512;
constexpr size_t KR_SMEM_BUDGET = 200 * 1024;
constexpr int KR_BATCH = 4;  // loads issued before their stores in the copy loops

struct KronArgs {
    const void* a;
    const float* r1;  // [in] or null (ones)
    const float* q1;  // [n1][n1]
    const float* q2;  // [n2][n2]
    const float* r2;  // [in / d] or null (ones)
    const float* M;   // [d][D]
    void* u;
    int a_bf16, u_bf16;
    int batch, in, n1, n2, d, D, K;
    int C, R, Rp, NT;  // CTAs per token group, rows per CTA (Rp: padded to even), tokens per group
    int n2p, ldq;      // n2 rounded up to 4; row stride of Q2 in shared memory (floats, ldq / 4 odd)
};

// Shared-memory carve-up (byte offsets, 16-byte aligned), strides in floats:
//   q2s [n2][ldq]        Q2 rows, zero columns n2 .. n2p
//   q1s [Rp][n1]         this CTA's rows of Q1 (zero padding rows)
//   xs  [NT][n1][n2p]    r1 o X of the group's tokens, later the compact Y [NT][R * n2]
//   ws  [NT][Rp][n2p]    W = Q1[own rows] X, zero columns n2 .. n2p
//   ms  [d][D]           M
struct KronLayout {
    size_t q2s, q1s, xs, ws, ms, total;
};

__host__ __device__ inline KronLayout kron_layout(const KronArgs& p) {
    KronLayout L;
    size_t off = 0;
    auto take = [&off](size_t bytes) {
        const size_t o = off;
        off += (bytes + 15) & ~size_t(15);
        return o;
    };
    L.q2s = take((size_t)p.n2 * p.ldq * 4);
    L.q1s = take((size_t)p.Rp * p.n1 * 4);
    L.xs = take((size_t)p.NT * p.n1 * p.n2p * 4);
    L.ws = take((size_t)p.NT * p.Rp * p.n2p * 4);
    L.ms = take((size_t)p.d * p.D * 4);
    L.total = off;
    return L;
}

// C_t[m][n] = sum_{k < K} A[m][k] * B_t[k][n] (t < nb, m < Mp, n < N): A rows at
// stride lda, B_t = B + t * bstr rows at stride ldb. A warp's work unit is TM rows
// x 32 consecutive columns, one column per lane: B reads are consecutive words
// (conflict-free), A reads are warp-wide broadcasts -- four contraction steps per
// float4 when AV4 (K and lda multiples of 4), which cuts the shared-memory
// wavefronts per FMA instruction from 5/4 to 12/32 at TM = 8.
template <int TM, bool AV4, class Store>
__device__ __forceinline__ void smem_gemm_ab(const float* A, int lda, const float* B, int ldb, size_t bstr, int nb,
                                             int Mp, int N, int K, Store store) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = (N + 31) >> 5, mg = Mp / TM;
    const int per_t = mg * nblk;
    for (int unit = warp; unit < nb * per_t; unit += KR_THREADS / 32) {
        const int t = unit / per_t, rem = unit - t * per_t;
        const int g = rem / nblk, n = (rem - g * nblk) * 32 + lane;
        const bool live = n < N;
        const float* a = A + (size_t)g * TM * lda;
        const float* b = B + (size_t)t * bstr + (live ? n : 0);
        float acc0[TM], acc1[TM];
#pragma unroll
        for (int i = 0; i < TM; ++i) acc0[i] = acc1[i] = 0.f;
        int k = 0;
        if (AV4) {
            for (; k < K; k += 4) {
                const float b0 = b[(size_t)k * ldb], b1 = b[(size_t)(k + 1) * ldb];
                const float b2 = b[(size_t)(k + 2) * ldb], b3 = b[(size_t)(k + 3) * ldb];
#pragma unroll
                for (int i = 0; i < TM; ++i) {
                    const float4 av = *reinterpret_cast<const float4*>(a + (size_t)i * lda + k);
                    acc0[i] = fmaf(av.x, b0, acc0[i]);
                    acc1[i] = fmaf(av.y, b1, acc1[i]);
                    acc0[i] = fmaf(av.z, b2, acc0[i]);
                    acc1[i] = fmaf(av.w, b3, acc1[i]);
                }
            }
        }
#pragma unroll 2
        for (; k + 1 < K; k += 2) {
            const float b0 = b[(size_t)k * ldb], b1 = b[(size_t)(k + 1) * ldb];
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                acc0[i] = fmaf(a[(size_t)i * lda + k], b0, acc0[i]);
                acc1[i] = fmaf(a[(size_t)i * lda + k + 1], b1, acc1[i]);
            }
        }
        if (k < K) {
            const float b0 = b[(size_t)k * ldb];
#pragma unroll
            for (int i = 0; i < TM; ++i) acc0[i] = fmaf(a[(size_t)i * lda + k], b0, acc0[i]);
        }
        if (live) {
#pragma unroll
            for (int i = 0; i < TM; ++i) store(t, g * TM + i, n, acc0[i] + acc1[i]);
        }
    }
}

// C_t[m][n] = sum_{k < Kp} A_t[m][k] * B[n][k] (t < nb, m < Mp, n < N): A_t = A +
// t * astr rows at stride lda, B rows at stride ldb (Kp, lda, ldb multiples of 4;
// ldb / 4 odd). Units of TM rows x 32 consecutive columns; lanes read consecutive
// B rows in float4 (conflict-free) and share the A rows (broadcast).
template <int TM, class Store>
__device__ __forceinline__ void smem_gemm_abt(const float* A, int lda, size_t astr, const float* B, int ldb, int nb,
                                              int Mp, int N, int Kp, Store store) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = (N + 31) >> 5, mg = Mp / TM;
    const int per_t = mg * nblk;
    for (int unit = warp; unit < nb * per_t; unit += KR_THREADS / 32) {
        const int t = unit / per_t, rem = unit - t * per_t;
        const int g = rem / nblk, n = (rem - g * nblk) * 32 + lane;
        const bool live = n < N;
        const float* a = A + (size_t)t * astr + (size_t)g * TM * lda;
        const float* b = B + (size_t)(live ? n : 0) * ldb;
        float acc0[TM], acc1[TM];
#pragma unroll
        for (int i = 0; i < TM; ++i) acc0[i] = acc1[i] = 0.f;
#pragma unroll 2
        for (int k = 0; k < Kp; k += 4) {
            const float4 bv = *reinterpret_cast<const float4*>(b + k);
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const float4 av = *reinterpret_cast<const float4*>(a + (size_t)i * lda + k);
                acc0[i] = fmaf(av.x, bv.x, acc0[i]);
                acc1[i] = fmaf(av.y, bv.y, acc1[i]);
                acc0[i] = fmaf(av.z, bv.z, acc0[i]);
                acc1[i] = fmaf(av.w, bv.w, acc1[i]);
            }
        }
        if (live) {
#pragma unroll
            for (int i = 0; i < TM; ++i) store(t, g * TM + i, n, acc0[i] + acc1[i]);
        }
    }
}

// WIDE: the multi-token (prefill) instantiation with 8-row tiles; the decode
// instantiation leaves them out and keeps its register count low.
template <bool WIDE>
__global__ void __launch_bounds__(KR_THREADS, 1) lift_kron_kernel(const KronArgs p) {
    // the next kernel on the stream may be scheduled early; it reads u only
    // after its own griddepcontrol.wait, which waits for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(16) uint8_t kr_smem[];
    const int c = (int)(blockIdx.x % p.C);  // row slice of the token group
    const int row0 = c * p.R;
    const int tid = threadIdx.x;
    const KronLayout L = kron_layout(p);
    float* q2s = reinterpret_cast<float*>(kr_smem + L.q2s);
    float* q1s = reinterpret_cast<float*>(kr_smem + L.q1s);
    float* xs = reinterpret_cast<float*>(kr_smem + L.xs);
    float* ws = reinterpret_cast<float*>(kr_smem + L.ws);
    float* ms = reinterpret_cast<float*>(kr_smem + L.ms);
    // row-by-quad copies: thread (tr, tx) takes quad tx of rows tr, tr + rstep, ...
    const bool vec = (p.n2 & 3) == 0;
    const int nq = p.n2p >> 2;
    const int tr = tid / nq, tx = tid - tr * nq, rstep = KR_THREADS / nq;

    // factors first: they do not depend on the kernel before this one, and stay
    // in shared memory for every token group this CTA takes
    if (vec && tr < rstep) {
        for (int r0 = tr; r0 < p.n2; r0 += KR_BATCH * rstep) {
            float4 v[KR_BATCH];
#pragma unroll
            for (int k = 0; k < KR_BATCH; ++k) {
                const int r = r0 + k * rstep;
                if (r < p.n2) v[k] = __ldg(reinterpret_cast<const float4*>(p.q2 + (size_t)r * p.n2) + tx);
            }
#pragma unroll
            for (int k = 0; k < KR_BATCH; ++k) {
                const int r = r0 + k * rstep;
                if (r < p.n2) *reinterpret_cast<float4*>(q2s + (size_t)r * p.ldq + 4 * tx) = v[k];
            }
        }
    } else if (!vec) {
        for (int idx = tid; idx < p.n2 * p.n2p; idx += KR_THREADS) {
            const int i2 = idx / p.n2p, j2 = idx - i2 * p.n2p;
            q2s[(size_t)i2 * p.ldq + j2] = j2 < p.n2 ? __ldg(p.q2 + (size_t)i2 * p.n2 + j2) : 0.f;
        }
    }
    for (int idx = tid; idx < p.Rp * p.n1; idx += KR_THREADS) {
        const int r = idx / p.n1, j1 = idx - r * p.n1;
        q1s[idx] = r < p.R ? __ldg(p.q1 + (size_t)(row0 + r) * p.n1 + j1) : 0.f;
    }
    for (int idx = tid; idx < p.d * p.D; idx += KR_THREADS) ms[idx] = __ldg(p.M + idx);
    if (p.n2p > p.n2) {  // contraction padding of W: never overwritten
        const int pad = p.n2p - p.n2;
        for (int idx = tid; idx < p.NT * p.Rp * pad; idx += KR_THREADS) {
            const int row = idx / pad;
            ws[(size_t)row * p.n2p + p.n2 + (idx - row * pad)] = 0.f;
        }
    }

    // the activations are written by the kernel before this one on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int ngroups = (p.batch + p.NT - 1) / p.NT;
    const int gstride = (int)(gridDim.x / p.C);
    const int nblk = p.R * p.n2 / p.d;  // d-blocks in this CTA's rows
    const int blk0 = row0 * p.n2 / p.d;
    const int ycs = p.R * p.n2;         // compact Y of one token: y[t][r * n2 + i2], kept in xs
    const int nbs = KR_THREADS / p.D;   // lift: thread (ljb, lj) takes column lj of blocks ljb, ljb + nbs, ...
    const int lj = tid % p.D, ljb = tid / p.D;
    const bool tm4 = (p.Rp & 3) == 0;
    // multi-token groups (prefill): 8-row tiles, Q1 read four steps per float4
    const bool wide = WIDE && (p.Rp & 7) == 0 && (p.n1 & 3) == 0;
    for (int grp = (int)(blockIdx.x / p.C); grp < ngroups; grp += gstride) {
        const int tok0 = grp * p.NT;

        // r1 o X: all n1 rows of the group's tokens (zero rows for missing tokens)
        if (vec) {
            if (tr < rstep) {
                for (int t = 0; t < p.NT; ++t) {
                    const int tok = tok0 + t;
                    float* xt = xs + (size_t)t * p.n1 * p.n2p;
                    for (int r0 = tr; r0 < p.n1; r0 += KR_BATCH * rstep) {
                        float4 v[KR_BATCH];
#pragma unroll
                        for (int k = 0; k < KR_BATCH; ++k) {
                            const int r = r0 + k * rstep;
                            v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (r < p.n1 && tok < p.batch) {
                                const long long e = (long long)r * p.n2 + 4 * tx;
                                v[k] = load_act4(p.a, p.a_bf16, (long long)tok * p.in + e, (long long)p.batch * p.in);
                                if (p.r1) {
                                    const float4 w = __ldg(reinterpret_cast<const float4*>(p.r1 + e));
                                    v[k].x *= w.x;
                                    v[k].y *= w.y;
                                    v[k].z *= w.z;
                                    v[k].w *= w.w;
                                }
                            }
                        }
#pragma unroll
                        for (int k = 0; k < KR_BATCH; ++k) {
                            const int r = r0 + k * rstep;
                            if (r < p.n1) *reinterpret_cast<float4*>(xt + (size_t)r * p.n2p + 4 * tx) = v[k];
                        }
                    }
                }
            }
        } else {
            for (int idx = tid; idx < p.NT * p.n1 * p.n2p; idx += KR_THREADS) {
                const int j2 = idx % p.n2p, row = idx / p.n2p;  // row = t * n1 + r
                const int tok = tok0 + row / p.n1, r = row % p.n1;
                float v = 0.f;
                if (j2 < p.n2 && tok < p.batch) {
                    const long long e = (long long)r * p.n2 + j2;
                    v = load_act(p.a, p.a_bf16, (long long)tok * p.in + e, (long long)p.batch * p.in);
                    if (p.r1) v *= __ldg(p.r1 + e);
                }
                xs[idx] = v;
            }
        }
        __syncthreads();

        // 1. W_t = Q1[own rows] X_t
        auto store_w = [&](int t, int m, int n, float v) { ws[((size_t)t * p.Rp + m) * p.n2p + n] = v; };
        if (wide)
            smem_gemm_ab<8, true>(q1s, p.n1, xs, p.n2p, (size_t)p.n1 * p.n2p, p.NT, p.Rp, p.n2, p.n1, store_w);
        else if (tm4)
            smem_gemm_ab<4, false>(q1s, p.n1, xs, p.n2p, (size_t)p.n1 * p.n2p, p.NT, p.Rp, p.n2, p.n1, store_w);
        else
            smem_gemm_ab<2, false>(q1s, p.n1, xs, p.n2p, (size_t)p.n1 * p.n2p, p.NT, p.Rp, p.n2, p.n1, store_w);
        __syncthreads();

        // 2. Y_t = W_t Q2^T, compact into xs (X is no longer needed)
        auto store_y = [&](int t, int m, int n, float v) {
            if (m < p.R) xs[(size_t)t * ycs + (size_t)m * p.n2 + n] = v;
        };
        if (wide)
            smem_gemm_abt<8>(ws, p.n2p, (size_t)p.Rp * p.n2p, q2s, p.ldq, p.NT, p.Rp, p.n2, p.n2p, store_y);
        else if (tm4)
            smem_gemm_abt<4>(ws, p.n2p, (size_t)p.Rp * p.n2p, q2s, p.ldq, p.NT, p.Rp, p.n2, p.n2p, store_y);
        else
            smem_gemm_abt<2>(ws, p.n2p, (size_t)p.Rp * p.n2p, q2s, p.ldq, p.NT, p.Rp, p.n2, p.n2p, store_y);
        __syncthreads();

        // 3. lift the d-blocks of this CTA's rows: u[tok][b D + j] = r2[b] sum_i M[i][j] a'[b d + i]
        if (ljb < nbs) {
            for (int t = 0; t < p.NT; ++t) {
                const int tok = tok0 + t;
                if (tok >= p.batch) break;
                const float* yt = xs + (size_t)t * ycs;
                for (int b = ljb; b < nblk; b += nbs) {
                    const float* yb = yt + b * p.d;
                    float acc = 0.f;
#pragma unroll 4
                    for (int i = 0; i < p.d; ++i) acc = fmaf(ms[i * p.D + lj], yb[i], acc);
                    const float sc = p.r2 ? __ldg(p.r2 + blk0 + b) : 1.f;
                    store_u(p.u, p.u_bf16, (long long)tok * p.K + (long long)(blk0 + b) * p.D + lj, (long long)p.batch * p.K, sc * acc);
                }
            }
        }
        // lifted coordinates past (in / d) * D are zero
        if (c == p.C - 1) {
            const int k0 = p.in / p.d * p.D, pad = p.K - k0;
            for (int it = tid; it < p.NT * pad; it += KR_THREADS) {
                const int t = it / pad, k = k0 + (it - t * pad);
                if (tok0 + t < p.batch) store_u(p.u, p.u_bf16, (long long)(tok0 + t) * p.K + k, (long long)p.batch * p.K, 0.f);
            }
        }
        __syncthreads();  // Y has been read before the next group's X overwrites it
    }
}

// Decode batches (<= 32 tokens): C CTAs per token, C the largest of 16, 8, 4, 2,
// 1 with n1 % C == 0 and (n1 / C) * n2 a multiple of d. Larger batches: whole
// tokens per CTA (C = 1), NT of them (4, 2 or 1, while the shared memory fits).
bool kron_plan(int batch, int n1, int n2, int d, int D, KronArgs& p, size_t& smem) {
    p.n1 = n1;
    p.n2 = n2;
    p.d = d;
    p.D = D;
    p.n2p = (n2 + 3) & ~3;
    p.ldq = p.n2p % 8 == 0 ? p.n2p + 4 : p.n2p;
    int C = 1;
    if (batch <= 32)
        for (int cand = 16; cand >= 1; cand >>= 1)
            if (n1 % cand == 0 && ((n1 / cand) * n2) % d == 0) {
                C = cand;
                break;
            }
    if (((n1 / C) * n2) % d != 0) return false;
    p.C = C;
    p.R = n1 / C;
    p.Rp = p.R + (p.R & 1);
    for (int NT = batch <= 32 ? 1 : 4;; NT >>= 1) {
        p.NT = NT;
        smem = kron_layout(p).total;
        if (smem <= KR_SMEM_BUDGET || NT == 1) break;
    }
    return smem <= KR_SMEM_BUDGET;
}

}  // namespace

bool lift_kron_supported(int batch, int in, int n1, int n2, int d, int D) {
    KronArgs p;
    size_t smem = 0;
    (void)in;
    return kron_plan(batch, n1, n2, d, D, p, smem);
}

cudaError_t launch_lift_kron(const void* a, bool a_bf16, int batch, int in, const float* r1, const float* q1,
                             int n1, const float* q2, int n2, const float* r2, const float* M, int d, int D,
                             void* u, bool u_bf16, int K, cudaStream_t st) {
    KronArgs p;
    size_t smem = 0;
    if (!kron_plan(batch, n1, n2, d, D, p, smem)) return cudaErrorInvalidValue;
    p.a = a;
    p.r1 = r1;
    p.q1 = q1;
    p.q2 = q2;
    p.r2 = r2;
    p.M = M;
    p.u = u;
    p.a_bf16 = a_bf16;
    p.u_bf16 = u_bf16;
    p.batch = batch;
    p.in = in;
    p.K = K;
    static size_t granted[64] = {};
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (dev >= 64 || granted[dev] < smem) {
        cudaError_t e = cudaFuncSetAttribute(lift_kron_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)KR_SMEM_BUDGET);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(lift_kron_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)KR_SMEM_BUDGET);
        if (e != cudaSuccess) return e;
        if (dev < 64) granted[dev] = KR_SMEM_BUDGET;
    }
    // decode: every token group at once; large batches: persistent CTAs, as many
    // as are resident (512 threads x 128 registers: one per SM)
    const int ngroups = (batch + p.NT - 1) / p.NT;
    const int groups_at_once = batch <= 32 ? ngroups : std::max(1, std::min(ngroups, sms / p.C));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(groups_at_once * p.C), 1, 1);
    cfg.blockDim = dim3(KR_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return p.NT > 1 ? cudaLaunchKernelEx(&cfg, lift_kron_kernel<true>, p)
                    : cudaLaunchKernelEx(&cfg, lift_kron_kernel<false>, p);
}

}  // namespace lq

LQ_DEBUG_FLAG_TAKE(debug_take_lift_kron)
