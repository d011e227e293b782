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
// One thread-block cluster of C CTAs covers NT tokens; CTA c owns rows
// [c R, (c + 1) R) of X (R = n1 / C) for all NT tokens:
//   1. Z = (r1 o X) Q2^T on its rows (rows are independent), kept transposed;
//   2. cluster barrier, then every CTA gathers all of Z^T from the cluster's
//      shared memory (distributed shared memory loads);
//   3. Y = Q1[own rows] Z;
//   4. a' = r2 o Y and the lift of the d-blocks inside its rows (C is chosen
//      so that R * n2 is a multiple of d: no block straddles two CTAs).
// A last cluster barrier keeps each CTA's Z alive until every peer has read it.
// Both products read their operands along the contraction index in float4:
// Q1, Q2 and the activations in their natural row-major layout, Z transposed.
// All arithmetic is fp32 (fp32 accumulation of n2 and then n1 products).
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "lq_internal.h"
#include "lq_lift_common.cuh"

namespace lq {
namespace {

namespace cg = cooperative_groups;

constexpr int KR_THREADS = 512;
constexpr size_t KR_SMEM_BUDGET = 200 * 1024;

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
    int C, R, Rp, NT;            // CTAs per cluster, rows per CTA (Rp: padded), tokens per cluster
    int n1p, n2p, ldq, ldz, lda2;  // padded widths and shared-memory row strides (floats)
};

// Shared-memory carve-up (byte offsets, 16-byte aligned), strides in floats:
//   q2s [n2][ldq]         Q2 rows, zero columns n2 .. n2p
//   q1s [Rp][n1p]         this CTA's rows of Q1, zero padding
//   xy  [NT][Rp][n2p]     r1 o X (zero padding), later Y
//   zt  [NT][n2][ldz]     Z^T of this CTA's rows: zt[t][i2][r] (read by the whole cluster)
//   za  [NT][n2][lda2]    Z^T of all rows: za[t][i2][j1], zero columns n1 .. n1p
//   ms  [d][D]            M
// ldq / 4 and lda2 / 4 are odd: consecutive threads reading consecutive rows
// in float4 hit distinct banks.
struct KronLayout {
    size_t q2s, q1s, xy, zt, za, ms, total;
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
    L.q1s = take((size_t)p.Rp * p.n1p * 4);
    L.xy = take((size_t)p.NT * p.Rp * p.n2p * 4);
    L.zt = take((size_t)p.NT * p.n2 * p.ldz * 4);
    L.za = take((size_t)p.NT * p.n2 * p.lda2 * 4);
    L.ms = take((size_t)p.d * p.D * 4);
    L.total = off;
    return L;
}

// C_t[m][n] = sum_{k < Kp} A_t[m][k] * B_t[n][k] for t < nb, m < Mp, n < N, with
// A_t = A + t * astr, B_t = B + t * bstr (rows at stride lda / ldb; Kp, lda, ldb
// multiples of 4; Mp a multiple of TM). Work units of one warp: TM rows x 32
// consecutive columns, one column per lane, so lanes read consecutive B rows
// (conflict-free with ldb / 4 odd) and share the A rows (broadcast reads).
// store(t, m, n, value) receives each result.
template <int TM, class Store>
__device__ __forceinline__ void smem_gemm_abt(const float* A, int lda, size_t astr, const float* B, int ldb,
                                              size_t bstr, int nb, int Mp, int N, int Kp, Store store) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = (N + 31) >> 5, mg = Mp / TM;
    const int per_t = mg * nblk;
    for (int unit = warp; unit < nb * per_t; unit += KR_THREADS / 32) {
        const int t = unit / per_t, rem = unit - t * per_t;
        const int g = rem / nblk, n = (rem - g * nblk) * 32 + lane;
        const bool live = n < N;
        const float* a = A + (size_t)t * astr + (size_t)g * TM * lda;
        const float* b = B + (size_t)t * bstr + (size_t)(live ? n : 0) * ldb;
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

template <class Store>
__device__ __forceinline__ void gemm_abt(const float* A, int lda, size_t astr, const float* B, int ldb, size_t bstr,
                                         int nb, int Mp, int N, int Kp, Store store) {
    if (Mp % 4 == 0)
        smem_gemm_abt<4>(A, lda, astr, B, ldb, bstr, nb, Mp, N, Kp, store);
    else
        smem_gemm_abt<2>(A, lda, astr, B, ldb, bstr, nb, Mp, N, Kp, store);
}

constexpr int KR_BATCH = 4;  // loads issued before their stores in the copy loops

__global__ void __launch_bounds__(KR_THREADS, 1) lift_kron_kernel(const KronArgs p) {
    // the next kernel on the stream may be scheduled early; it reads u only
    // after its own griddepcontrol.wait, which waits for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(16) uint8_t kr_smem[];
    cg::cluster_group cl = cg::this_cluster();
    const int c = (int)cl.block_rank();
    const int row0 = c * p.R;  // first row of X owned by this CTA
    const int tid = threadIdx.x;
    const KronLayout L = kron_layout(p);
    float* q2s = reinterpret_cast<float*>(kr_smem + L.q2s);
    float* q1s = reinterpret_cast<float*>(kr_smem + L.q1s);
    float* xy = reinterpret_cast<float*>(kr_smem + L.xy);
    float* zt = reinterpret_cast<float*>(kr_smem + L.zt);
    float* za = reinterpret_cast<float*>(kr_smem + L.za);
    float* ms = reinterpret_cast<float*>(kr_smem + L.ms);
    // row-by-quad copies: thread (tr, tx) takes quad tx of rows tr, tr + rstep, ...
    const bool vec = (p.n2 & 3) == 0;
    const int nq = p.n2p >> 2;
    const int tr = tid / nq, tx = tid - tr * nq, rstep = KR_THREADS / nq;

    // factors first: they do not depend on the kernel before this one, and stay
    // in shared memory for every token group this cluster takes
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
    for (int idx = tid; idx < p.Rp * p.n1p; idx += KR_THREADS) {
        const int r = idx / p.n1p, j1 = idx - r * p.n1p;
        q1s[idx] = r < p.R && j1 < p.n1 ? __ldg(p.q1 + (size_t)(row0 + r) * p.n1 + j1) : 0.f;
    }
    for (int idx = tid; idx < p.d * p.D; idx += KR_THREADS) ms[idx] = __ldg(p.M + idx);
    if (p.n1p > p.n1) {  // contraction padding of the gathered Z^T: never overwritten
        const int pad = p.n1p - p.n1;
        for (int idx = tid; idx < p.NT * p.n2 * pad; idx += KR_THREADS) {
            const int row = idx / pad;
            za[(size_t)row * p.lda2 + p.n1 + (idx - row * pad)] = 0.f;
        }
    }

    // the activations are written by the kernel before this one on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int ngroups = (p.batch + p.NT - 1) / p.NT;
    const int nclusters = (int)(gridDim.x / p.C);
    const int nblk = p.R * p.n2 / p.d;  // d-blocks in this CTA's rows
    const int blk0 = row0 * p.n2 / p.d;
    const int ycs = p.R * p.n2;         // compact Y of one token: yc[t][r * n2 + i2]
    const int nbs = KR_THREADS / p.D;   // lift: thread (ljb, lj) takes column lj of blocks ljb, ljb + nbs, ...
    const int lj = tid % p.D, ljb = tid / p.D;
    for (int grp = (int)(blockIdx.x / p.C); grp < ngroups; grp += nclusters) {
        const int tok0 = grp * p.NT;

        // r1 o X for this CTA's rows of the group's tokens (zero padding)
        if (vec) {
            if (tr < rstep) {
                for (int t = 0; t < p.NT; ++t) {
                    const int tok = tok0 + t;
                    float* xt = xy + (size_t)t * p.Rp * p.n2p;
                    for (int r0 = tr; r0 < p.Rp; r0 += KR_BATCH * rstep) {
                        float4 v[KR_BATCH];
#pragma unroll
                        for (int k = 0; k < KR_BATCH; ++k) {
                            const int r = r0 + k * rstep;
                            v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (r < p.R && tok < p.batch) {
                                const long long e = (long long)(row0 + r) * p.n2 + 4 * tx;
                                v[k] = load_act4(p.a, p.a_bf16, (long long)tok * p.in + e);
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
                            if (r < p.Rp) *reinterpret_cast<float4*>(xt + (size_t)r * p.n2p + 4 * tx) = v[k];
                        }
                    }
                }
            }
        } else {
            for (int idx = tid; idx < p.NT * p.Rp * p.n2p; idx += KR_THREADS) {
                const int j2 = idx % p.n2p, row = idx / p.n2p;
                const int r = row % p.Rp, tok = tok0 + row / p.Rp;
                float v = 0.f;
                if (r < p.R && j2 < p.n2 && tok < p.batch) {
                    const long long e = (long long)(row0 + r) * p.n2 + j2;
                    v = load_act(p.a, p.a_bf16, (long long)tok * p.in + e);
                    if (p.r1) v *= __ldg(p.r1 + e);
                }
                xy[idx] = v;
            }
        }
        __syncthreads();

        // 1. Z_t = (r1 o X_t) Q2^T on this CTA's rows, stored transposed: zt[t][i2][r]
        gemm_abt(xy, p.n2p, (size_t)p.Rp * p.n2p, q2s, p.ldq, 0, p.NT, p.Rp, p.n2, p.n2p,
                 [&](int t, int m, int n, float v) { zt[((size_t)t * p.n2 + n) * p.ldz + m] = v; });
        cl.sync();  // every CTA's rows of Z are complete and visible to the cluster

        // 2. gather Z^T of all n1 rows: columns [peer R, (peer + 1) R) live in CTA peer
        if ((p.R & 3) == 0) {
            const int rq = p.R >> 2, gr = tid / rq, gx = tid - gr * rq, gstep = KR_THREADS / rq;
            if (gr < gstep) {
                for (int row = gr; row < p.NT * p.n2; row += gstep) {  // row = t * n2 + i2
                    float4 v[8];
#pragma unroll
                    for (int peer = 0; peer < 8; ++peer)
                        if (peer < p.C)
                            v[peer] = *reinterpret_cast<const float4*>(cl.map_shared_rank(zt, peer) +
                                                                       (size_t)row * p.ldz + 4 * gx);
#pragma unroll
                    for (int peer = 0; peer < 8; ++peer)
                        if (peer < p.C)
                            *reinterpret_cast<float4*>(za + (size_t)row * p.lda2 + peer * p.R + 4 * gx) = v[peer];
                }
            }
        } else {
            const int per_peer = p.NT * p.n2 * p.R;
            for (int q = tid; q < p.C * per_peer; q += KR_THREADS) {
                const int peer = q / per_peer, rem = q - peer * per_peer;
                const int x = rem % p.R, row = rem / p.R;
                za[(size_t)row * p.lda2 + peer * p.R + x] = cl.map_shared_rank(zt, peer)[(size_t)row * p.ldz + x];
            }
        }
        __syncthreads();

        // 3. Y_t = Q1[own rows] Z_t, compact into xy (X is no longer needed)
        gemm_abt(q1s, p.n1p, 0, za, p.lda2, (size_t)p.n2 * p.lda2, p.NT, p.Rp, p.n2, p.n1p,
                 [&](int t, int m, int n, float v) {
                     if (m < p.R) xy[(size_t)t * ycs + (size_t)m * p.n2 + n] = v;
                 });
        __syncthreads();

        // 4. lift the d-blocks of this CTA's rows: u[tok][b D + j] = r2[b] sum_i M[i][j] a'[b d + i]
        if (ljb < nbs) {
            for (int t = 0; t < p.NT; ++t) {
                const int tok = tok0 + t;
                if (tok >= p.batch) break;
                const float* yt = xy + (size_t)t * ycs;
                for (int b = ljb; b < nblk; b += nbs) {
                    const float* yb = yt + b * p.d;
                    float acc = 0.f;
#pragma unroll 4
                    for (int i = 0; i < p.d; ++i) acc = fmaf(ms[i * p.D + lj], yb[i], acc);
                    const float sc = p.r2 ? __ldg(p.r2 + blk0 + b) : 1.f;
                    store_u(p.u, p.u_bf16, (long long)tok * p.K + (long long)(blk0 + b) * p.D + lj, sc * acc);
                }
            }
        }
        // lifted coordinates past (in / d) * D are zero
        if (c == p.C - 1) {
            const int k0 = p.in / p.d * p.D, pad = p.K - k0;
            for (int it = tid; it < p.NT * pad; it += KR_THREADS) {
                const int t = it / pad, k = k0 + (it - t * pad);
                if (tok0 + t < p.batch) store_u(p.u, p.u_bf16, (long long)(tok0 + t) * p.K + k, 0.f);
            }
        }
        // peers have finished reading this CTA's Z^T, and every thread is done
        // with Y, before the next group overwrites them
        cl.sync();
    }
}

// Decode batches (<= 32 tokens): one token per cluster of C CTAs, C the largest
// of 8, 4, 2, 1 with n1 % C == 0 and (n1 / C) * n2 a multiple of d, so a token
// is spread over C SMs. Larger batches: whole tokens per CTA (C = 1), NT of
// them per CTA (4, 2 or 1, while the shared memory fits), so that no work is
// split that need not be.
bool kron_plan(int batch, int n1, int n2, int d, int D, KronArgs& p, size_t& smem) {
    int C = 1;
    if (batch <= 32)
        for (int cand = 8; cand >= 1; cand >>= 1)
            if (n1 % cand == 0 && ((n1 / cand) * n2) % d == 0) {
                C = cand;
                break;
            }
    if (((n1 / C) * n2) % d != 0) return false;
    p.n1 = n1;
    p.n2 = n2;
    p.d = d;
    p.D = D;
    p.C = C;
    p.R = n1 / C;
    p.Rp = p.R + (p.R & 1);
    p.n1p = (n1 + 3) & ~3;
    p.n2p = (n2 + 3) & ~3;
    p.ldq = p.n2p % 8 == 0 ? p.n2p + 4 : p.n2p;
    p.lda2 = p.n1p % 8 == 0 ? p.n1p + 4 : p.n1p;
    p.ldz = (p.Rp + 3) & ~3;
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
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || granted[dev] < smem) {
        cudaError_t e =
            cudaFuncSetAttribute(lift_kron_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KR_SMEM_BUDGET);
        if (e != cudaSuccess) return e;
        if (dev < 64) granted[dev] = KR_SMEM_BUDGET;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(KR_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    // persistent clusters: as many as are resident at once (each loops over
    // token groups with the factors kept in shared memory)
    static int cached_key[64][3] = {};
    const int ngroups = (batch + p.NT - 1) / p.NT;
    int resident = 0;
    if (dev < 64 && cached_key[dev][0] == p.C && cached_key[dev][1] == (int)smem) {
        resident = cached_key[dev][2];
    } else {
        cfg.gridDim = dim3((unsigned)p.C, 1, 1);
        if (cudaOccupancyMaxActiveClusters(&resident, lift_kron_kernel, &cfg) != cudaSuccess) {
            cudaGetLastError();
            resident = 0;
        }
        if (dev < 64 && resident > 0) {
            cached_key[dev][0] = p.C;
            cached_key[dev][1] = (int)smem;
            cached_key[dev][2] = resident;
        }
    }
    if (resident < 1) resident = 1;
    cfg.gridDim = dim3((unsigned)(std::min(ngroups, resident) * p.C), 1, 1);
    return cudaLaunchKernelEx(&cfg, lift_kron_kernel, p);
}

}  // namespace lq
