// Encoder: weights -> 1-bit lifted codes (LiftQuant paper note, "Key designs" 2).
//
// Each block w of d consecutive weights of a row is represented by the sign
// pattern y in {+-1}^D whose codeword M y is nearest to w. The page replaces the
// naive 2^D search by a pseudo-inverse start plus a search over an auxiliary
// vector of D - d coordinates (2^{D-d} patterns). Read as:
//   candidate 0:      y = sign(M^+ w), M^+ = M^T (M M^T)^{-1};
//   candidate 1 + p:  the first D - d coordinates are the pattern p (bit a set
//                     <=> +1), the last d solve M_B y_B = w - M_A z and are
//                     rounded: y_B = sign(M_B^{-1} (w - M_A z));
// sign(0) = +1; the smallest ||w - M y||^2 wins, the earliest candidate on ties.
//
// The search is an offline step whose result is an integer code, so it runs in
// float64. Each CTA inverts M M^T and M_B once (parallel Gauss-Jordan in shared
// memory); the (row, block) units are spread over every warp of the grid. The 32
// lanes of a warp split the 2^{D-d} patterns of its block and walk their share in
// Gray-code order, so each step flips one auxiliary coordinate and updates
// v = w - M_A z, r = M_B^{-1} v and q = M_B y_B incrementally (O(d) per step
// instead of O(d D)); a warp reduction picks the minimum. The pattern's D bits
// are ORed into the (zeroed) words of the 32-per-word layout that lq_gemv reads;
// a block's bits can straddle three words, shared with its neighbours.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "lq_debug.cuh"
#include "lq_internal.h"

namespace lq {
namespace {

constexpr int EN_THREADS = 256;
constexpr int EN_WARPS = EN_THREADS / 32;

struct EncArgs {
    const float* w;    // [rows][in]
    const float* M;    // [d][D]
    uint32_t* packed;  // [rows][K/32]
    float* err;        // [rows][in/d] or null
    int rows, in, d, D, K, nblk;
};

// Shared memory (8-byte units): Md [d][D], P [D][d] = M^T (M M^T)^{-1},
// Bi [d][d] = M_B^{-1}, G [d][D-d] = M_B^{-1} M_A, gi [d][d] (M M^T, then M_B,
// as inputs of the inversions), work [d][2d], fac [d] and one flag word.
struct EncLayout {
    size_t md, pm, bi, g, gi, wk, fac, flag, total;
};

__host__ __device__ inline EncLayout enc_layout(int d, int D) {
    EncLayout L;
    size_t off = 0;
    auto take = [&off](size_t n8) {
        const size_t o = off;
        off += n8 * 8;
        return o;
    };
    L.md = take((size_t)d * D);
    L.pm = take((size_t)D * d);
    L.bi = take((size_t)d * d);
    L.g = take((size_t)d * (D - d) + 1);
    L.gi = take((size_t)d * d);
    L.wk = take((size_t)d * 2 * d);
    L.fac = take((size_t)d);
    L.flag = take(1);
    L.total = off;
    return L;
}

// inv = A^{-1} (n x n, row-major, shared memory) by Gauss-Jordan elimination with
// partial pivoting on [A | I]; every thread of the block takes part. Sets *flag
// when a pivot is zero (the matrix is singular).
__device__ void gj_inverse(const double* A, double* inv, double* wk, double* fac, int n, int* flag) {
    const int n2 = 2 * n;
    for (int idx = threadIdx.x; idx < n * n2; idx += EN_THREADS) {
        const int r = idx / n2, k = idx - r * n2;
        wk[idx] = k < n ? A[r * n + k] : (k - n == r ? 1.0 : 0.0);
    }
    __syncthreads();
    for (int c = 0; c < n; ++c) {
        if (threadIdx.x == 0) {
            int piv = c;
            for (int r = c + 1; r < n; ++r)
                if (fabs(wk[r * n2 + c]) > fabs(wk[piv * n2 + c])) piv = r;
            if (wk[piv * n2 + c] == 0.0) {
                *flag = 1;
            } else if (piv != c) {
                for (int k = 0; k < n2; ++k) {
                    const double t = wk[c * n2 + k];
                    wk[c * n2 + k] = wk[piv * n2 + k];
                    wk[piv * n2 + k] = t;
                }
            }
        }
        __syncthreads();
        if (*flag) return;  // uniform: every thread reads the flag after the barrier
        const double pivot = wk[c * n2 + c];
        __syncthreads();
        for (int k = threadIdx.x; k < n2; k += EN_THREADS) wk[c * n2 + k] /= pivot;
        __syncthreads();
        for (int r = threadIdx.x; r < n; r += EN_THREADS) fac[r] = wk[r * n2 + c];
        __syncthreads();
        for (int idx = threadIdx.x; idx < n * n2; idx += EN_THREADS) {
            const int r = idx / n2, k = idx - r * n2;
            if (r != c) wk[idx] -= fac[r] * wk[c * n2 + k];
        }
        __syncthreads();
    }
    for (int idx = threadIdx.x; idx < n * n; idx += EN_THREADS) {
        const int r = idx / n, k = idx - r * n;
        inv[idx] = wk[r * n2 + n + k];
    }
    __syncthreads();
}

template <int MAXD>
__device__ __forceinline__ double sqdist(const double (&v)[MAXD], const double (&q)[MAXD], int d) {
    double e = 0.0;
#pragma unroll
    for (int i = 0; i < MAXD; ++i)
        if (i < d) {
            const double t = v[i] - q[i];
            e = fma(t, t, e);
        }
    return e;
}

// One block of d weights, one warp: returns (in every lane) the chosen pattern
// and its squared error.
template <int MAXD>
__device__ void encode_block(const double* Md, const double* P, const double* Bi, const double* G, int d, int D,
                             const float* wb, int lane, uint64_t& y_out, double& e_out) {
    const int na = D - d;
    double w[MAXD];
#pragma unroll
    for (int i = 0; i < MAXD; ++i) w[i] = i < d ? (double)__ldg(wb + i) : 0.0;

    // candidate 0: the pseudo-inverse start y0 = sign(M^+ w); lane j holds coordinates j, j + 32
    uint64_t y0 = 0;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int j = lane + 32 * half;
        bool pos = false;
        if (j < D) {
            double acc = 0.0;
#pragma unroll
            for (int i = 0; i < MAXD; ++i)
                if (i < d) acc = fma(P[j * d + i], w[i], acc);
            pos = acc >= 0.0;
        }
        y0 |= (uint64_t)__ballot_sync(0xffffffffu, pos) << (32 * half);
    }
    double e0 = 0.0;
#pragma unroll
    for (int i = 0; i < MAXD; ++i)
        if (i < d) {
            double res = w[i];
            for (int j = 0; j < D; ++j) res -= Md[i * D + j] * (((y0 >> j) & 1ull) ? 1.0 : -1.0);
            e0 = fma(res, res, e0);
        }

    // candidates 1 + p: lane takes Gray-code indices [i0, i0 + per) of the 2^{D-d} patterns
    const uint32_t total = 1u << na;
    const uint32_t per = total >= 32 ? total >> 5 : 1u;
    const uint32_t i0 = (uint32_t)lane * per;
    double best_e = __longlong_as_double(0x7ff0000000000000ll);  // +inf
    uint32_t best_p = 0xffffffffu, best_yb = 0;
    if (i0 < total) {
        uint32_t g = i0 ^ (i0 >> 1);
        double v[MAXD], r[MAXD], q[MAXD];
#pragma unroll
        for (int i = 0; i < MAXD; ++i) {
            double acc = w[i];
            if (i < d)
                for (int a = 0; a < na; ++a) acc -= Md[i * D + a] * (((g >> a) & 1u) ? 1.0 : -1.0);
            v[i] = acc;  // v = w - M_A z
        }
        uint32_t yb = 0;
#pragma unroll
        for (int k = 0; k < MAXD; ++k) {
            double acc = 0.0;
            if (k < d) {
#pragma unroll
                for (int i = 0; i < MAXD; ++i)
                    if (i < d) acc = fma(Bi[k * d + i], v[i], acc);
                if (acc >= 0.0) yb |= 1u << k;
            }
            r[k] = acc;  // r = M_B^{-1} v
        }
#pragma unroll
        for (int i = 0; i < MAXD; ++i) {
            double acc = 0.0;
            if (i < d) {
#pragma unroll
                for (int k = 0; k < MAXD; ++k)
                    if (k < d) acc += Md[i * D + na + k] * (((yb >> k) & 1u) ? 1.0 : -1.0);
            }
            q[i] = acc;  // q = M_B y_B
        }
        best_e = sqdist(v, q, d);
        best_p = g;
        best_yb = yb;
        for (uint32_t s = 1; s < per; ++s) {
            const int a = __ffs(i0 + s) - 1;  // consecutive Gray codes differ in this bit
            g ^= 1u << a;
            const double delta = ((g >> a) & 1u) ? 2.0 : -2.0;  // z_a moved by delta
#pragma unroll
            for (int i = 0; i < MAXD; ++i)
                if (i < d) {
                    v[i] = fma(-delta, Md[i * D + a], v[i]);
                    r[i] = fma(-delta, G[i * na + a], r[i]);
                }
            uint32_t nyb = 0;
#pragma unroll
            for (int k = 0; k < MAXD; ++k)
                if (k < d && r[k] >= 0.0) nyb |= 1u << k;
            uint32_t ch = nyb ^ yb;
            while (ch) {
                const int k = __ffs(ch) - 1;
                ch &= ch - 1;
                const double sg = ((nyb >> k) & 1u) ? 2.0 : -2.0;
#pragma unroll
                for (int i = 0; i < MAXD; ++i)
                    if (i < d) q[i] = fma(sg, Md[i * D + na + k], q[i]);
            }
            yb = nyb;
            const double e = sqdist(v, q, d);
            if (e < best_e || (e == best_e && g < best_p)) {
                best_e = e;
                best_p = g;
                best_yb = yb;
            }
        }
    }
    // smallest error over the warp, the lowest pattern on ties
#pragma unroll
    for (int off = 16; off; off >>= 1) {
        const double oe = __shfl_xor_sync(0xffffffffu, best_e, off);
        const uint32_t op = __shfl_xor_sync(0xffffffffu, best_p, off);
        const uint32_t oy = __shfl_xor_sync(0xffffffffu, best_yb, off);
        if (oe < best_e || (oe == best_e && op < best_p)) {
            best_e = oe;
            best_p = op;
            best_yb = oy;
        }
    }
    if (e0 <= best_e) {  // candidate 0 comes first
        y_out = y0;
        e_out = e0;
    } else {
        y_out = (uint64_t)best_p | ((uint64_t)best_yb << na);
        e_out = best_e;
    }
}

template <int MAXD>
__global__ void __launch_bounds__(EN_THREADS, 1) encode_kernel(const EncArgs p) {
    extern __shared__ __align__(16) uint8_t en_smem[];
    const int d = p.d, D = p.D, na = D - d;
    const EncLayout L = enc_layout(d, D);
    double* Md = reinterpret_cast<double*>(en_smem + L.md);
    double* P = reinterpret_cast<double*>(en_smem + L.pm);
    double* Bi = reinterpret_cast<double*>(en_smem + L.bi);
    double* G = reinterpret_cast<double*>(en_smem + L.g);
    double* gi = reinterpret_cast<double*>(en_smem + L.gi);
    double* wk = reinterpret_cast<double*>(en_smem + L.wk);
    double* fac = reinterpret_cast<double*>(en_smem + L.fac);
    int* flag = reinterpret_cast<int*>(en_smem + L.flag);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // M in float64, M^+ = M^T (M M^T)^{-1}, M_B^{-1} and M_B^{-1} M_A, once per CTA
    for (int idx = tid; idx < d * D; idx += EN_THREADS) Md[idx] = (double)__ldg(p.M + idx);
    if (tid == 0) *flag = 0;
    __syncthreads();
    for (int idx = tid; idx < d * d; idx += EN_THREADS) {
        const int i = idx / d, k = idx - i * d;
        double acc = 0.0;
        for (int j = 0; j < D; ++j) acc = fma(Md[i * D + j], Md[k * D + j], acc);
        gi[idx] = acc;
    }
    __syncthreads();
    gj_inverse(gi, Bi, wk, fac, d, flag);  // Bi holds (M M^T)^{-1} for now
    if (!*flag) {
        for (int idx = tid; idx < D * d; idx += EN_THREADS) {
            const int j = idx / d, i = idx - j * d;
            double acc = 0.0;
            for (int k = 0; k < d; ++k) acc = fma(Md[k * D + j], Bi[k * d + i], acc);
            P[idx] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < d * d; idx += EN_THREADS) {
            const int i = idx / d, k = idx - i * d;
            gi[idx] = Md[i * D + na + k];
        }
        __syncthreads();
        gj_inverse(gi, Bi, wk, fac, d, flag);
        if (!*flag) {
            for (int idx = tid; idx < d * na; idx += EN_THREADS) {
                const int i = idx / na, a = idx - i * na;
                double acc = 0.0;
                for (int k = 0; k < d; ++k) acc = fma(Bi[i * d + k], Md[k * D + a], acc);
                G[idx] = acc;
            }
        }
    }
    __syncthreads();
    const bool singular = *flag != 0;

    const int nq = p.K / 32;
    const long long units = (long long)p.rows * p.nblk;
    for (long long u = (long long)blockIdx.x * EN_WARPS + warp; u < units; u += (long long)gridDim.x * EN_WARPS) {
        const int row = (int)(u / p.nblk), b = (int)(u - (long long)row * p.nblk);
        uint64_t y = 0;
        double e = __longlong_as_double(0x7ff8000000000000ll);  // NaN: singular M M^T or M_B
        const bool w_ok = LQ_IN_BOUNDS((long long)row * p.in + (long long)b * d + d - 1, (long long)p.rows * p.in);
        if (!singular && w_ok)
            encode_block<MAXD>(Md, P, Bi, G, d, D, p.w + (long long)row * p.in + (long long)b * d, lane, y, e);
        if (lane == 0) {
            if (p.err && LQ_IN_BOUNDS(u, units)) p.err[u] = (float)e;
            // bits [b D, b D + D) of the row: words q, q + 1 and (past 64 bits) q + 2
            uint32_t* words = p.packed + (long long)row * nq;
            const long long bit0 = (long long)b * D;
            const int q = (int)(bit0 >> 5), o = (int)(bit0 & 31);
            const uint64_t sh = y << o;
            const uint32_t w0 = (uint32_t)sh, w1 = (uint32_t)(sh >> 32), w2 = o ? (uint32_t)(y >> (64 - o)) : 0u;
            // every word a block touches lies within its own row (K / 32 words)
            if (w0 && LQ_IN_BOUNDS(q, nq)) atomicOr(words + q, w0);
            if (w1 && LQ_IN_BOUNDS(q + 1, nq)) atomicOr(words + q + 1, w1);
            if (w2 && LQ_IN_BOUNDS(q + 2, nq)) atomicOr(words + q + 2, w2);
        }
    }
}

}  // namespace

size_t encode_smem(int d, int D) { return enc_layout(d, D).total; }

template <int MAXD>
cudaError_t launch_encode_t(const EncArgs& p, size_t smem, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<MAXD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_kernel<MAXD>, EN_THREADS, smem) != cudaSuccess ||
        per_sm < 1) {
        cudaGetLastError();
        per_sm = 1;
    }
    const long long units = (long long)p.rows * p.nblk;
    const long long need = (units + EN_WARPS - 1) / EN_WARPS;
    const int grid = (int)std::max(1ll, std::min(need, (long long)sms * per_sm));
    encode_kernel<MAXD><<<grid, EN_THREADS, smem, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_encode(const float* w, int rows, int in, const float* M, int d, int D, uint32_t* packed, int K,
                          float* err, cudaStream_t st) {
    EncArgs p;
    p.w = w;
    p.M = M;
    p.packed = packed;
    p.err = err;
    p.rows = rows;
    p.in = in;
    p.d = d;
    p.D = D;
    p.K = K;
    p.nblk = in / d;
    const size_t smem = enc_layout(d, D).total;
    // the kernel ORs each block's bits into its words
    cudaError_t e = cudaMemsetAsync(packed, 0, (size_t)rows * (K / 32) * sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    if (d <= 8) return launch_encode_t<8>(p, smem, st);
    if (d <= 10) return launch_encode_t<10>(p, smem, st);
    if (d <= 12) return launch_encode_t<12>(p, smem, st);
    if (d <= 16) return launch_encode_t<16>(p, smem, st);
    return launch_encode_t<24>(p, smem, st);
}

}  // namespace lq

LQ_DEBUG_FLAG_TAKE(debug_take_encode)
