// Decode 1-bit GEMV, batch 1..16 (LiftQuant paper note, "Key designs" 4: after
// the small matmul T* a the layer is a 1-bit x float matmul with W_q, then
// diag(s)):
//
//   o[c][r] = s[r] * sum_k sigma[r][k] u[c][k],   sigma = +1 if the bit is set.
//
// Design (integer tensor-core operands, exact accumulation):
//   * sum_k sigma u = 2 sum_{bit=1} u - sum_k u, so only the set bits matter.
//   * quantize_kernel turns each K-part of u into 24-bit fixed point with a
//     per-part, per-column power-of-two scale (|u_q| <= 2^22, so an element's
//     rounding error is at most 2^-22 of the part maximum) and writes three
//     balanced int8 digit planes u_q = d0 + 2^8 d1 + 2^16 d2 (the bytes of
//     (u_q + 0x808080) ^ 0x808080) to the workspace, once per call.
//   * gemv_kernel: a sign word w yields eight u8 operand registers
//     w & (0x01010101 << j), j = 0..7: bytes 0 or 2^j for bits j, j+8, j+16,
//     j+24 -- one LOP3 per four weights, nothing unpacked to memory. These are
//     the A fragments of mma.sync m16n8k32 u8 x s8 -> s32. (Measured on B200:
//     0.5 such MMA per clock per SM = 256 weight bits/clk/SM, above the ~186
//     bits/clk/SM that saturate HBM; tcgen05 kind::i8 with N <= 64 sustains one
//     MMA per ~46 clocks = 90 bits/clk/SM, too slow at decode batch sizes.)
//     B fragments are the digit planes (column n = 3c + p), read through L1.
//     One s32 accumulator set per j keeps the 2^j scales apart; every integer
//     sum is exact.
//   * About one CTA per SM. A CTA owns G groups of 16 rows; each group's K is
//     split into H parts, one warp per (group, part), so 12-16 warps keep the
//     SM busy. Each warp streams its 16 rows through a private ring of 1 KB
//     TMA tiles (16 rows x 64 bytes: conflict-free fragment reads), one mbarrier
//     per stage, every wait bounded. The H partial sums of a group are added in
//     fixed order through shared memory: deterministic results.
//   * The GEMV is launched as a programmatic dependent of the quantizer: its
//     CTAs start their weight streams while u is being quantized and wait
//     (griddepcontrol.wait) only before the first digit read.
//   * Rows whose word count is not a multiple of 4 (not 16-byte aligned for
//     TMA) use guarded register loads instead of the ring.
// Batches above 8 run as two column passes over the weights.
#include <cuda.h>

#include <algorithm>

#include "lq_internal.h"
#include "lq_sm100.cuh"

namespace lq {
namespace {

constexpr int kMaxCols = 8;       // batch columns per GEMV pass
constexpr int kMaxBatch = 16;
constexpr int kMaxParts = 8;      // K-parts per row group
constexpr int kMaxWarps = 16;
constexpr int kStepWords = 16;    // words per row a warp consumes per step
constexpr int kStageBytes = 16 * kStepWords * 4;  // 16 rows x 64 bytes
constexpr int kQThreads = 256;

struct QMeta {
    long long sall;  // sum of u_q over the part
    int F;           // u_q = rint(u * 2^F)
    int pad;
};

// Workspace: digit planes uint32 [3*batch][kwp][8] (kwp = kw rounded up to 16;
// byte i of word (n, x, j) is digit n%3 of u[n/3][32x + j + 8i]), then QMeta
// [batch][kMaxParts] at a 256-byte boundary.
__host__ __device__ inline size_t digits_bytes(int kw, int batch) {
    const size_t kwp = (size_t)(kw + 15) / 16 * 16;
    return (size_t)3 * batch * kwp * 32;
}
__host__ __device__ inline size_t meta_offset(int kw, int batch) { return (digits_bytes(kw, batch) + 255) / 256 * 256; }

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 load_words(const uint32_t* row, int x, int kw) {
    uint4 v;
    v.x = x < kw ? __ldg(row + x) : 0u;
    v.y = x + 1 < kw ? __ldg(row + x + 1) : 0u;
    v.z = x + 2 < kw ? __ldg(row + x + 2) : 0u;
    v.w = x + 3 < kw ? __ldg(row + x + 3) : 0u;
    return v;
}

// 2^e as a float for -126 <= e <= 127.
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// Exponent e with cmax < 2^e (frexp convention) from the bits of cmax >= 0;
// zero and subnormal maxima use e = -126.
__device__ __forceinline__ int max_exponent(int cmax_bits) {
    const int E = (cmax_bits >> 23) & 255;
    return E == 0 ? -126 : E - 126;
}

// ---------------------------------------------------------------- quantizer
struct QArgs {
    const float* u;  // [batch][K]
    uint32_t* digits;
    QMeta* meta;
    int K, kw, kwp, batch, kp;  // kp: words per part
};

// One CTA per (part h, column c).
__global__ void __launch_bounds__(kQThreads) quantize_kernel(const QArgs q) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // let the GEMV start streaming weights
    __shared__ float redf[kQThreads / 32];
    __shared__ long long redl[kQThreads / 32];
    const int h = blockIdx.x, c = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int x0 = h * q.kp;
    const int x1 = min(q.kwp, x0 + q.kp);      // digits are written up to the padded width
    const int x1v = min(q.kw, x0 + q.kp);      // ... from u entries below K
    const float* uc = q.u + (long long)c * q.K;

    float mx = 0.f;
    for (int i = 32 * x0 / 4 + threadIdx.x; i < 32 * x1v / 4; i += kQThreads) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(uc) + i);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) redf[warp] = mx;
    __syncthreads();
    mx = redf[0];
#pragma unroll
    for (int w = 1; w < kQThreads / 32; ++w) mx = fmaxf(mx, redf[w]);
    const int F = 22 - max_exponent(__float_as_int(mx));  // mx * 2^F < 2^22
    const float sa = pow2f(F >> 1), sb = pow2f(F - (F >> 1));

    long long qsum = 0;
    for (int x = x0 + threadIdx.x; x < x1; x += kQThreads) {
        uint32_t tb[32];  // balanced digits of element e in the bytes of tb[e]
        if (x < x1v) {
            const float4* src = reinterpret_cast<const float4*>(uc + 32 * x);
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
                const float4 v = __ldg(src + qq);
                const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int qi = __float2int_rn((f[i] * sa) * sb);
                    qsum += qi;
                    tb[4 * qq + i] = (uint32_t)(qi + 0x808080) ^ 0x808080u;
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) tb[e] = 0u;
        }
#pragma unroll
        for (int pl = 0; pl < 3; ++pl) {
            const uint32_t sel = (uint32_t)pl | ((uint32_t)(pl + 4) << 4);
            uint32_t P[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                // byte i of P[j] = digit pl of element j + 8 i
                const uint32_t lo = __byte_perm(tb[j], tb[j + 8], sel);
                const uint32_t hi = __byte_perm(tb[j + 16], tb[j + 24], sel);
                P[j] = __byte_perm(lo, hi, 0x5410);
            }
            uint4* dst = reinterpret_cast<uint4*>(q.digits + ((long long)(3 * c + pl) * q.kwp + x) * 8);
            dst[0] = make_uint4(P[0], P[1], P[2], P[3]);
            dst[1] = make_uint4(P[4], P[5], P[6], P[7]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) qsum += __shfl_xor_sync(0xffffffffu, qsum, off);
    if (lane == 0) redl[warp] = qsum;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long s = 0;
        for (int w = 0; w < kQThreads / 32; ++w) s += redl[w];
        QMeta m;
        m.sall = s;
        m.F = F;
        m.pad = 0;
        q.meta[c * kMaxParts + h] = m;
    }
}

// ---------------------------------------------------------------- GEMV
struct GemvArgs {
    const uint32_t* packed;
    const float* s;
    const uint32_t* digits;
    const QMeta* meta;
    float* o;         // [batch][out]
    unsigned* status;
    int out, kw, kwp;
    int c0, ncols;    // columns [c0, c0 + ncols) in this pass
    int G, H, kp;     // row groups per CTA, K-parts per group, words per part
};

__host__ __device__ inline size_t gemv_smem(int G, int H, int ncols, int stages, bool tma) {
    const int W = G * H;
    const size_t ring = tma ? (size_t)W * stages * kStageBytes : 0;
    const size_t bars = tma ? (size_t)W * stages * 8 : 0;
    const size_t part = (size_t)W * ncols * 16 * 8;
    return ring + bars + part + 16;
}

template <int NG, int STAGES, bool TMA>
__global__ void __launch_bounds__(NG == 3 ? 256 : 512, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tmap, const GemvArgs p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int W = p.G * p.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int gi = warp / p.H, h = warp - gi * p.H;
    const int m0 = blockIdx.x * 16 * p.G;
    const int wrow0 = m0 + 16 * gi;
    const int x_begin = h * p.kp;
    const int x_end = min(p.kw, x_begin + p.kp);
    const int steps = max(0, x_end - x_begin + kStepWords - 1) / kStepWords;
    const int ndig = 3 * p.ncols;

    uint8_t* ring = smem + (size_t)warp * STAGES * kStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (TMA ? (size_t)W * STAGES * kStageBytes : 0)) + warp * STAGES;
    double* part = reinterpret_cast<double*>(smem + (TMA ? (size_t)W * STAGES * (kStageBytes + 8) : 0));

    if (TMA) {
        if (lane == 0) {
            for (int st = 0; st < STAGES; ++st) sm100::mbar_init(sm100::smem_addr(bars + st), 1);
            sm100::fence_barrier_init();
        }
        __syncwarp();
    }
    auto issue = [&](int w) {  // lane 0 only
        const int slot = w % STAGES;
        sm100::mbar_arrive_expect_tx(sm100::smem_addr(bars + slot), kStageBytes);
        sm100::tma_load_2d(sm100::smem_addr(ring + slot * kStageBytes), &tmap, x_begin + w * kStepWords, wrow0,
                           sm100::smem_addr(bars + slot));
    };
    int issued = 0;
    if (TMA && lane == 0) {
        for (; issued < STAGES - 1 && issued < steps; ++issued) issue(issued);
    }

    const int r0 = wrow0 + g, r1 = r0 + 8;
    const bool v0 = r0 < p.out, v1 = r1 < p.out;
    const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
    const uint32_t* row0 = p.packed + (long long)min(r0, p.out - 1) * p.kw;
    const uint32_t* row1 = p.packed + (long long)min(r1, p.out - 1) * p.kw;
    uint4 wa = zero4, wb = zero4;
    if (!TMA) {
        wa = v0 ? load_words(row0, x_begin + 4 * t, p.kw) : zero4;
        wb = v1 ? load_words(row1, x_begin + 4 * t, p.kw) : zero4;
    }

    // the digit planes come from the quantizer launched just before this kernel
    asm volatile("griddepcontrol.wait;" ::: "memory");

    int acc[NG][8][4];
#pragma unroll
    for (int n = 0; n < NG; ++n)
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[n][j][e] = 0;

    bool ok = true;
    for (int w = 0; w < steps && ok; ++w) {
        uint4 ca, cb;
        if (TMA) {
            const int slot = w % STAGES;
            if (!sm100::mbar_wait(sm100::smem_addr(bars + slot), (w / STAGES) & 1, p.status)) {
                ok = false;  // flagged in the status word; results of this call are invalid
                break;
            }
            const uint8_t* st = ring + slot * kStageBytes;
            ca = *reinterpret_cast<const uint4*>(st + g * 64 + t * 16);
            cb = *reinterpret_cast<const uint4*>(st + (g + 8) * 64 + t * 16);
            __syncwarp();  // every lane has read the slot refilled below in a later step
            if (lane == 0 && issued < steps) issue(issued++);
        } else {
            ca = wa;
            cb = wb;
            if (w + 1 < steps) {
                const int xn = x_begin + (w + 1) * kStepWords + 4 * t;
                wa = v0 ? load_words(row0, xn, p.kw) : zero4;
                wb = v1 ? load_words(row1, xn, p.kw) : zero4;
            }
        }
#pragma unroll
        for (int sg = 0; sg < 2; ++sg) {
            const int xg = x_begin + w * kStepWords + 4 * t + 2 * sg;  // word of k-columns 4t..4t+3
            uint32_t B[NG][16];
#pragma unroll
            for (int n = 0; n < NG; ++n) {
                const int col = 8 * n + g;
                if (col < ndig) {
                    const uint4* src =
                        reinterpret_cast<const uint4*>(p.digits + ((long long)(3 * p.c0 + col) * p.kwp + xg) * 8);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const uint4 v = __ldg(src + r);
                        B[n][4 * r + 0] = v.x;
                        B[n][4 * r + 1] = v.y;
                        B[n][4 * r + 2] = v.z;
                        B[n][4 * r + 3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < 16; ++r) B[n][r] = 0u;
                }
            }
            const uint32_t a_lo0 = sg ? ca.z : ca.x, a_hi0 = sg ? ca.w : ca.y;  // row g: words xg, xg+1
            const uint32_t a_lo1 = sg ? cb.z : cb.x, a_hi1 = sg ? cb.w : cb.y;  // row g+8
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t msk = 0x01010101u << j;
                const uint32_t a0 = a_lo0 & msk, a1 = a_lo1 & msk, a2 = a_hi0 & msk, a3 = a_hi1 & msk;
#pragma unroll
                for (int n = 0; n < NG; ++n) mma_u8s8(acc[n][j], a0, a1, a2, a3, B[n][j], B[n][8 + j]);
            }
        }
    }
    if (TMA) {
        // Leave nothing in flight: on the normal path every issued tile was waited
        // for; after a timeout, wait (bounded) for the rest.
        if (lane == 0 && !ok)
            for (int w = issued - (STAGES - 1) < 0 ? 0 : issued - (STAGES - 1); w < issued; ++w)
                sm100::mbar_wait(sm100::smem_addr(bars + w % STAGES), (w / STAGES) & 1, p.status);
        __syncwarp();
    }

    // ---- combine the eight 2^j accumulators: V = sum_j 2^(7-j) acc_j = 2^7 sum_k bit*d
    // V lives in this warp's own ring (1 KB * NG <= STAGES KB) or, without a ring,
    // in its partial-sum slot area reused after the gather below.
    __shared__ double vsm_fallback[1];  // never used with a ring; keeps the pointer well-defined
    double* V = TMA ? reinterpret_cast<double*>(ring) : vsm_fallback;
    double vreg[NG][4];
#pragma unroll
    for (int n = 0; n < NG; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            long long v = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) v += (long long)acc[n][j][e] * (1ll << (7 - j));
            vreg[n][e] = (double)v;
        }
    double* out_part = part + (size_t)warp * p.ncols * 16;  // [ncols][16 rows]
    if (TMA) {
#pragma unroll
        for (int n = 0; n < NG; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) V[(g + 8 * (e >> 1)) * (8 * NG) + 8 * n + 2 * t + (e & 1)] = vreg[n][e];
        __syncwarp();
        for (int item = lane; item < 16 * p.ncols; item += 32) {
            const int row = item & 15, c = item >> 4;
            const double* vr = V + row * (8 * NG) + 3 * c;
            const QMeta mt = p.meta[(p.c0 + c) * kMaxParts + h];
            // 2^7 sum_{bit=1} u_q (exact in double); sum_k sigma u_q = 2 sum_{bit=1} u_q - sum_k u_q
            const double s1 = vr[0] + 256.0 * vr[1] + 65536.0 * vr[2];
            const double unscale = __longlong_as_double((long long)(1023 - mt.F) << 52);
            out_part[c * 16 + row] = (s1 * (1.0 / 64.0) - (double)mt.sall) * unscale;
        }
    } else {
        // without a ring: exchange the plane columns through shuffles, one column at a time
        for (int c = 0; c < p.ncols; ++c) {
            const QMeta mt = p.meta[(p.c0 + c) * kMaxParts + h];
            const double unscale = __longlong_as_double((long long)(1023 - mt.F) << 52);
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {  // rows g (hr = 0) and g + 8
                double s1 = 0.0;
#pragma unroll
                for (int pl = 0; pl < 3; ++pl) {
                    const int col = 3 * c + pl, n = col >> 3, src_t = (col & 7) >> 1, e = 2 * hr + (col & 1);
                    double mine = 0.0;
#pragma unroll
                    for (int nn = 0; nn < NG; ++nn)
#pragma unroll
                        for (int ee = 0; ee < 4; ++ee)
                            if (nn == n && ee == e) mine = vreg[nn][ee];
                    const double v = __shfl_sync(0xffffffffu, mine, (lane & ~3) | src_t);
                    s1 += (pl == 0 ? 1.0 : pl == 1 ? 256.0 : 65536.0) * v;
                }
                if (t == 0) out_part[c * 16 + g + 8 * hr] = (s1 * (1.0 / 64.0) - (double)mt.sall) * unscale;
            }
        }
    }
    __syncthreads();

    // ---- add the H parts of each row group in fixed order, scale, store
    if (h == 0) {
        for (int item = lane; item < 16 * p.ncols; item += 32) {
            const int row = item & 15, c = item >> 4;
            const int m = wrow0 + row;
            if (m < p.out) {
                double sum = 0.0;
                for (int hh = 0; hh < p.H; ++hh) sum += part[((size_t)(gi * p.H + hh) * p.ncols + c) * 16 + row];
                p.o[(long long)(p.c0 + c) * p.out + m] = (float)(sum * (double)__ldg(p.s + m));
            }
        }
    }
    (void)W;
}

// ---------------------------------------------------------------- host side
int num_sms() {
    static int sms[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && sms[dev]) return sms[dev];
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (dev < 64) sms[dev] = n;
    return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

struct Plan {
    int G, H, kp, stages;
};

Plan make_plan(int out, int kw, int ng) {
    const int sms = num_sms();
    const int groups = (out + 15) / 16;
    const int wmax = ng == 3 ? 8 : kMaxWarps;
    Plan pl;
    pl.G = std::max(1, std::min(wmax, (groups + sms - 1) / sms));
    pl.H = std::max(1, std::min(kMaxParts, wmax / pl.G));
    pl.H = std::min(pl.H, (kw + kStepWords - 1) / kStepWords);  // at least one step per part
    pl.kp = ((kw + pl.H - 1) / pl.H + kStepWords - 1) / kStepWords * kStepWords;
    pl.H = (kw + pl.kp - 1) / pl.kp;  // drop empty parts
    const int W = pl.G * pl.H;
    pl.stages = W <= 8 ? 8 : W <= 12 ? 6 : 4;
    return pl;
}

template <int NG, int STAGES, bool TMA>
cudaError_t launch_kernel(const CUtensorMap& map, const GemvArgs& p, cudaStream_t st) {
    const size_t smem = gemv_smem(p.G, p.H, p.ncols, STAGES, TMA);
    static size_t granted[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || granted[dev] < smem) {
        cudaError_t e = cudaFuncSetAttribute(gemv_kernel<NG, STAGES, TMA>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) granted[dev] = smem;
    }
    const int groups = (p.out + 15) / 16;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((groups + p.G - 1) / p.G, 1, 1);
    cfg.blockDim = dim3(32 * p.G * p.H, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<NG, STAGES, TMA>, map, p);
}

template <int NG>
cudaError_t launch_ng(const CUtensorMap& map, const GemvArgs& p, int stages, bool tma, cudaStream_t st) {
    if (!tma) return launch_kernel<NG, 4, false>(map, p, st);
    if (stages == 8) return launch_kernel<NG, 8, true>(map, p, st);
    if (stages == 6) return launch_kernel<NG, 6, true>(map, p, st);
    return launch_kernel<NG, 4, true>(map, p, st);
}

}  // namespace

size_t gemv_workspace_size(int out, int K, int batch) {
    (void)out;
    const int kw = K / 32;
    return meta_offset(kw, batch) + (size_t)batch * kMaxParts * sizeof(QMeta);
}

cudaError_t launch_gemv(const uint32_t* packed, const float* s, int out, int K, const float* u, int batch, float* o,
                        void* workspace, unsigned* status, cudaStream_t st) {
    const int kw = K / 32;
    const int kwp = (kw + 15) / 16 * 16;
    const bool tma = (kw % 4) == 0;  // TMA needs 16-byte row pitch
    // One plan for every pass (the quantizer's parts must match the GEMV's).
    const Plan pl = make_plan(out, kw, (3 * std::min(batch, kMaxCols) + 7) / 8);

    uint32_t* digits = static_cast<uint32_t*>(workspace);
    QMeta* meta = reinterpret_cast<QMeta*>(static_cast<uint8_t*>(workspace) + meta_offset(kw, batch));
    QArgs q;
    q.u = u;
    q.digits = digits;
    q.meta = meta;
    q.K = K;
    q.kw = kw;
    q.kwp = kwp;
    q.batch = batch;
    q.kp = pl.kp;
    quantize_kernel<<<dim3(pl.H, batch), kQThreads, 0, st>>>(q);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    if (tma) {
        EncodeTiledFn encode = encode_fn();
        if (!encode) return cudaErrorNotSupported;
        cuuint64_t gdim[2] = {(cuuint64_t)kw, (cuuint64_t)out};
        cuuint64_t gstride[1] = {(cuuint64_t)kw * 4};
        cuuint32_t box[2] = {kStepWords, 16};
        cuuint32_t estride[2] = {1, 1};
        if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(packed), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    for (int c0 = 0; c0 < batch; c0 += kMaxCols) {
        GemvArgs p;
        p.packed = packed;
        p.s = s;
        p.digits = digits;
        p.meta = meta;
        p.o = o;
        p.status = status;
        p.out = out;
        p.kw = kw;
        p.kwp = kwp;
        p.c0 = c0;
        p.ncols = std::min(kMaxCols, batch - c0);
        p.G = pl.G;
        p.H = pl.H;
        p.kp = pl.kp;
        const int ng = (3 * p.ncols + 7) / 8;
        e = ng == 1 ? launch_ng<1>(map, p, pl.stages, tma, st)
            : ng == 2 ? launch_ng<2>(map, p, pl.stages, tma, st)
                      : launch_ng<3>(map, p, pl.stages, tma, st);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace lq
