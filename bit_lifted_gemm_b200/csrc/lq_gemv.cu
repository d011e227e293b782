// Decode 1-bit GEMV, batch 1..16 (LiftQuant paper note, "Key designs" 4: after
// the small matmul T* a the layer is a 1-bit x float matmul with W_q, then
// diag(s)):
//
//   o[c][r] = s[r] * sum_k sigma[r][k] u[c][k],   sigma = +1 if the bit is set.
//
// Design (integer tensor-core operands, exact accumulation):
//   * sum_k sigma u = 2 sum_{bit=1} u - sum_k u, so only the set bits matter.
//   * Each K-part of u becomes 24-bit fixed point with a per-part, per-column
//     power-of-two scale (|u_q| <= 2^22: an element's rounding error is at most
//     2^-22 of the part maximum), held as three balanced int8 digit planes
//     u_q = d0 + 2^8 d1 + 2^16 d2 -- the bytes of (u_q + 0x808080) ^ 0x808080.
//     Every CTA quantizes u for itself in its prologue, while its first weight
//     tiles are in flight; no workspace, no extra launch.
//   * A sign word w yields eight u8 operand registers w & (0x01010101 << j),
//     j = 0..7: bytes 0 or 2^j for bits j, j+8, j+16, j+24 -- one LOP3 per four
//     weights, nothing unpacked to memory. These are the A fragments of
//     mma.sync m16n8k32 u8 x s8 -> s32. (Measured on B200: 0.5 such MMA per
//     clock per SM = 256 weight bits/clk/SM in isolation, ~155 bits/clk/SM
//     with the LOP3s and fragment loads of this loop, against ~186 bits/clk/SM
//     that saturate HBM; tcgen05 kind::i8 with N <= 64 sustains one MMA per ~46
//     clocks = 90 bits/clk/SM, too slow at decode batch sizes.) B fragments are
//     the digit planes (MMA column n = 3c + p), read from shared memory where
//     word x sits at 16-byte chunk 2x + x/4 (a bank skew) with the (j, x),
//     (j, x+1) digits interleaved, so one conflict-free 16-byte load yields two
//     aligned B register pairs. One s32 accumulator set per j keeps the 2^j
//     scales apart; every integer sum is exact.
//   * About one CTA per SM. A CTA owns G groups of 16 rows; each group's K is
//     split into H parts, one warp per (group, part), so 12-16 warps keep the
//     SM busy. Each warp streams its 16 rows through a private ring of 1 KB TMA
//     tiles (16 rows x 64 bytes: conflict-free fragment reads), one mbarrier
//     per stage, every wait bounded. The H partial sums of a group are added in
//     fixed order through shared memory: deterministic results.
//   * The GEMV is launched as a programmatic dependent of whatever precedes it
//     on the stream (normally the activation lift): it starts its weight
//     streams early and waits (griddepcontrol.wait) only before reading u.
//   * Up to two batch columns per pass (six digit planes fill one n8 MMA tile);
//     larger batches run several passes. K is covered by one launch when the
//     digit planes fit in shared memory, else by several launches that add into
//     o in stream order. Rows whose word count is not a multiple of 4 (not
//     16-byte aligned for TMA) use guarded register loads instead of the ring.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "lq_internal.h"
#include "lq_sm100.cuh"

namespace lq {
namespace {

constexpr int kMaxParts = 8;      // K-parts per row group
constexpr int kMaxWarps = 16;
constexpr int kMaxColsPass = 2;   // batch columns per pass (6 digit planes <= n8)
constexpr int kStepWords = 16;    // words per row a warp consumes per step
constexpr int kStageBytes = 16 * kStepWords * 4;  // 16 rows x 64 bytes
constexpr size_t kSmemBudget = 200 * 1024;

// Digit-plane storage: 16-byte chunks; word pair (x, x+1), x even, occupies the
// four chunks from 2x + x/4 holding (j, x), (j, x+1) for j = 0..7 in order.
__host__ __device__ __forceinline__ int chunkpos(int x) { return 2 * x + (x >> 2); }

// Chunks per plane for `words` words: covers chunkpos(words - 1) + 1 and is
// 4 (mod 8), which separates the planes a quarter-warp reads.
__host__ __device__ __forceinline__ int plane_pitch(int words) {
    int cp = 2 * words + words / 4 + 4;
    return cp % 8 == 4 ? cp : cp + 4;
}

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm(  // not volatile: the result is the only effect, so the compiler may interleave it
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
__device__ __forceinline__ int max_exponent(unsigned cmax_bits) {
    const int E = (cmax_bits >> 23) & 255;
    return E == 0 ? -126 : E - 126;
}

// 32 elements of word x of u (zeros past the end of K).
__device__ __forceinline__ void load_word(const float* uc, int x, int kw, float (&v)[32]) {
    if (x < kw) {
        const float4* src = reinterpret_cast<const float4*>(uc + 32 * x);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 f = __ldg(src + q);
            v[4 * q] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;
    }
}

// Digits of one word: P[pl][j] holds, in byte i, digit pl of element j + 8 i.
__device__ __forceinline__ void word_digits(const float (&v)[32], float sa, float sb, uint32_t (&P)[3][8],
                                            long long& qsum) {
    uint32_t tb[32];  // balanced digits of element e in the bytes of tb[e]
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int qi = __float2int_rn((v[e] * sa) * sb);
        qsum += qi;
        tb[e] = (uint32_t)(qi + 0x808080) ^ 0x808080u;
    }
#pragma unroll
    for (int pl = 0; pl < 3; ++pl) {
        const uint32_t sel = (uint32_t)pl | ((uint32_t)(pl + 4) << 4);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t lo = __byte_perm(tb[j], tb[j + 8], sel);
            const uint32_t hi = __byte_perm(tb[j + 16], tb[j + 24], sel);
            P[pl][j] = __byte_perm(lo, hi, 0x5410);
        }
    }
}

struct GemvArgs {
    const uint32_t* packed;
    const float* s;
    const float* u;   // [batch][K]
    float* o;         // [batch][out]
    unsigned* status;
    int out, K, kw;
    int c0, ncols;    // columns [c0, c0 + ncols) in this pass (ncols <= 2)
    int kx0, kwc;     // words [kx0, kx0 + kwc) of K in this launch; kx0, kwc multiples of 16
    int G, H, kp;     // row groups per CTA, K-parts per group, words per part (multiple of 16)
    int pitch;        // chunks per shared-memory digit plane
    int accumulate;   // 1: o += this launch's result
};

__host__ __device__ inline size_t gemv_smem(int G, int H, int ncols, int stages, int pitch, bool tma) {
    const int W = G * H;
    size_t s = tma ? (size_t)W * stages * (kStageBytes + 8) : 0;  // rings + their barriers
    s += (size_t)3 * ncols * pitch * 16 + 128;                     // digit planes + zero block
    s += (size_t)W * ncols * 16 * 8;                               // partial sums
    s += (size_t)kMaxColsPass * kMaxParts * (4 + 8);               // per (column, part) max and sum of u_q
    return s + 16;
}

template <int STAGES, bool TMA>
__global__ void __launch_bounds__(512, 1) gemv_kernel(const __grid_constant__ CUtensorMap tmap, const GemvArgs p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int W = p.G * p.H;
    const int nthreads = 32 * W;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int gi = warp / p.H, h = warp - gi * p.H;
    const int m0 = blockIdx.x * 16 * p.G;
    const int wrow0 = m0 + 16 * gi;
    const int xl_begin = h * p.kp;                                    // local word of this warp's part
    const int x_begin = p.kx0 + xl_begin;                             // global word
    const int x_end = min(min(p.kw, p.kx0 + p.kwc), x_begin + p.kp);
    const int steps = max(0, x_end - x_begin + kStepWords - 1) / kStepWords;
    const int ndig = 3 * p.ncols;

    uint8_t* ring = smem + (size_t)warp * STAGES * kStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (TMA ? (size_t)W * STAGES * kStageBytes : 0)) + warp * STAGES;
    uint4* bplanes = reinterpret_cast<uint4*>(smem + (TMA ? (size_t)W * STAGES * (kStageBytes + 8) : 0));
    uint4* bzero = bplanes + (size_t)ndig * p.pitch;  // 8 zero chunks: digits of idle MMA columns
    double* part = reinterpret_cast<double*>(bzero + 8);
    unsigned* colmax = reinterpret_cast<unsigned*>(part + (size_t)W * p.ncols * 16);       // [c][h]
    unsigned long long* sall = reinterpret_cast<unsigned long long*>(colmax + kMaxColsPass * kMaxParts);

    if (TMA && lane == 0)
        for (int st = 0; st < STAGES; ++st) sm100::mbar_init(sm100::smem_addr(bars + st), 1);
    if (TMA) sm100::fence_barrier_init();
    if (threadIdx.x < 8) bzero[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x < kMaxColsPass * kMaxParts) {
        colmax[threadIdx.x] = 0u;
        sall[threadIdx.x] = 0ull;
    }
    __syncthreads();

    auto issue = [&](int w) {  // lane 0 only
        const int slot = w & (STAGES - 1);
        sm100::mbar_arrive_expect_tx(sm100::smem_addr(bars + slot), kStageBytes);
        sm100::tma_load_2d(sm100::smem_addr(ring + slot * kStageBytes), &tmap, x_begin + w * kStepWords, wrow0,
                           sm100::smem_addr(bars + slot));
    };
    int issued = 0;
    if (TMA && lane == 0)
        for (; issued < STAGES - 1 && issued < steps; ++issued) issue(issued);

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

    // u is written by the kernel before this one on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- quantize this launch's slice of u: item = (column, word pair), key = c * H + part;
    // pass 1 takes the per-(column, part) maxima, pass 2 writes the digit planes
    const int npairs = p.kwc / 2;
    const int nitems = p.ncols * npairs;
    const int items_round = (nitems + nthreads - 1) / nthreads * nthreads;  // uniform trip count
    for (int it = threadIdx.x; it < items_round; it += nthreads) {
        const bool live = it < nitems;
        const int c = live ? it / npairs : 0, pr = it - c * npairs;
        const int xg = p.kx0 + 2 * pr;
        const float* uc = p.u + (long long)(p.c0 + c) * p.K;
        float a[32], b[32];
        load_word(uc, live ? xg : p.kw, p.kw, a);
        load_word(uc, live ? xg + 1 : p.kw, p.kw, b);
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fmaxf(fabsf(a[e]), fabsf(b[e])));
        const unsigned key = live ? (unsigned)(c * p.H + (2 * pr) / p.kp) : 0xffffffffu;
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        const unsigned gmax = __reduce_max_sync(peers, __float_as_uint(mx));  // non-negative: bits order like values
        if (live && lane == __ffs(peers) - 1) atomicMax(colmax + key, gmax);
    }
    __syncthreads();
    for (int it = threadIdx.x; it < items_round; it += nthreads) {
        const bool live = it < nitems;
        const int c = live ? it / npairs : 0, pr = it - c * npairs;
        const int xg = p.kx0 + 2 * pr;
        const unsigned key = live ? (unsigned)(c * p.H + (2 * pr) / p.kp) : 0xffffffffu;
        long long qsum = 0;
        if (live) {
            const int F = 22 - max_exponent(colmax[key]);  // part max * 2^F < 2^22
            const float sa = pow2f(F >> 1), sb = pow2f(F - (F >> 1));
            uint32_t P0[3][8], P1[3][8];
            const float* uc = p.u + (long long)(p.c0 + c) * p.K;  // second read: L1 hits
            float a[32];
            load_word(uc, xg, p.kw, a);
            word_digits(a, sa, sb, P0, qsum);
            load_word(uc, xg + 1, p.kw, a);
            word_digits(a, sa, sb, P1, qsum);
#pragma unroll
            for (int pl = 0; pl < 3; ++pl) {
                uint4* dst = bplanes + (size_t)(3 * c + pl) * p.pitch + chunkpos(2 * pr);
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    dst[r] = make_uint4(P0[pl][2 * r], P1[pl][2 * r], P0[pl][2 * r + 1], P1[pl][2 * r + 1]);
            }
        }
        // group sums of u_q (|item sum| < 2^29): split into 16-bit halves so the
        // 32-bit warp reductions cannot overflow
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        const unsigned lo = __reduce_add_sync(peers, (unsigned)(qsum & 0xffff));
        const int hi = (int)__reduce_add_sync(peers, (unsigned)(int)(qsum >> 16));
        if (live && lane == __ffs(peers) - 1)
            atomicAdd(sall + key, (unsigned long long)(((long long)hi << 16) + (long long)lo));
    }
    __syncthreads();

    int acc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0;

    auto mma_half = [&](uint32_t lo0, uint32_t hi0, uint32_t lo1, uint32_t hi1, const uint32_t (&B)[16]) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t msk = 0x01010101u << j;
            mma_u8s8(acc[j], lo0 & msk, lo1 & msk, hi0 & msk, hi1 & msk, B[2 * j], B[2 * j + 1]);
        }
    };
    // B fragments: this lane's digit column (or the zero block), words 4t.. of the
    // step; the B register pair (b0, b1) of j is (B[2j], B[2j+1]).
    const bool live_col = g < ndig;
    const uint4* bsrc = live_col ? bplanes + (size_t)g * p.pitch + chunkpos(xl_begin + 4 * t) : bzero;
    const int binc = live_col ? 36 : 0;  // chunkpos advances 36 chunks per 16-word step
    auto fetch_b = [&](int half, uint32_t (&B)[16]) {
        const uint4* src = bsrc + 4 * half;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint4 v = src[r];
            B[4 * r + 0] = v.x;
            B[4 * r + 1] = v.y;
            B[4 * r + 2] = v.z;
            B[4 * r + 3] = v.w;
        }
        if (half) bsrc += binc;
    };

    bool ok = true;
    if (TMA) {
        // Software-pipelined by half steps: the next half's digits (and, at step
        // boundaries, the next weight tile) are read before the current half's
        // LOP3s and MMAs are issued.
        const uint8_t* ring_lane = ring + g * 64 + t * 16;
        const uint32_t bar0 = sm100::smem_addr(bars);
        int slot = 0;
        uint32_t phase = 0;
        auto fetch_tile = [&](uint4& ca, uint4& cb) -> bool {
            const uint32_t bar = bar0 + 8 * slot;
            if (!sm100::mbar_try_wait(bar, phase) && !sm100::mbar_wait(bar, phase, p.status)) return false;
            const uint8_t* st = ring_lane + slot * kStageBytes;
            ca = *reinterpret_cast<const uint4*>(st);
            cb = *reinterpret_cast<const uint4*>(st + 8 * 64);
            __syncwarp();  // every lane has read the slot before lane 0 refills it
            if (lane == 0 && issued < steps) issue(issued++);
            slot = (slot + 1) & (STAGES - 1);
            phase ^= slot == 0;
            return true;
        };
        uint4 ca = zero4, cb = zero4;
        uint32_t Bc[16], Bn[16];
        if (steps > 0) {
            ok = fetch_tile(ca, cb);  // flagged in the status word on timeout; results invalid
            fetch_b(0, Bc);
        }
        for (int w = 0; ok && w < steps; ++w) {
            fetch_b(1, Bn);
            mma_half(ca.x, ca.y, cb.x, cb.y, Bc);
            const uint32_t lo0 = ca.z, hi0 = ca.w, lo1 = cb.z, hi1 = cb.w;
            if (w + 1 < steps) {
                ok = fetch_tile(ca, cb);
                fetch_b(0, Bc);
            }
            mma_half(lo0, hi0, lo1, hi1, Bn);
        }
        // Leave nothing in flight: on the normal path every issued tile was waited
        // for; after a timeout, wait (bounded) for the rest.
        if (lane == 0 && !ok)
            for (int w = issued - (STAGES - 1) < 0 ? 0 : issued - (STAGES - 1); w < issued; ++w)
                sm100::mbar_wait(sm100::smem_addr(bars + (w & (STAGES - 1))), (w / STAGES) & 1, p.status);
        __syncwarp();
    } else {
        for (int w = 0; w < steps; ++w) {
            const uint4 ca = wa, cb = wb;
            if (w + 1 < steps) {
                const int xn = x_begin + (w + 1) * kStepWords + 4 * t;
                wa = v0 ? load_words(row0, xn, p.kw) : zero4;
                wb = v1 ? load_words(row1, xn, p.kw) : zero4;
            }
            uint32_t B[16];
            fetch_b(0, B);
            mma_half(ca.x, ca.y, cb.x, cb.y, B);
            fetch_b(1, B);
            mma_half(ca.z, ca.w, cb.z, cb.w, B);
        }
    }

    // ---- combine the eight 2^j accumulators: V = sum_j 2^(7-j) acc_j = 2^7 sum_k bit*d,
    // then gather the three planes of each column with shuffles
    double vreg[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        long long v = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) v += (long long)acc[j][e] * (1ll << (7 - j));
        vreg[e] = (double)v;
    }
    double* out_part = part + (size_t)warp * p.ncols * 16;  // [ncols][16 rows]
    for (int c = 0; c < p.ncols; ++c) {
        const int key = c * p.H + h;
        const int F = 22 - max_exponent(colmax[key]);
        const double unscale = __longlong_as_double((long long)(1023 - F) << 52);
        const double sq = (double)(long long)sall[key];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {  // rows g (hr = 0) and g + 8
            double s1 = 0.0;
#pragma unroll
            for (int pl = 0; pl < 3; ++pl) {
                const int col = 3 * c + pl, e = 2 * hr + (col & 1);
                double mine = 0.0;
#pragma unroll
                for (int ee = 0; ee < 4; ++ee)
                    if (ee == e) mine = vreg[ee];
                const double v = __shfl_sync(0xffffffffu, mine, (lane & ~3) | (col >> 1));
                s1 += (pl == 0 ? 1.0 : pl == 1 ? 256.0 : 65536.0) * v;  // exact: 2^7 sum_{bit=1} u_q
            }
            // sum_k sigma u_q = 2 sum_{bit=1} u_q - sum_k u_q, then undo the 2^F scale
            if (t == 0) out_part[c * 16 + g + 8 * hr] = (s1 * (1.0 / 64.0) - sq) * unscale;
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
                float* dst = p.o + (long long)(p.c0 + c) * p.out + m;
                const float val = (float)(sum * (double)__ldg(p.s + m));
                *dst = p.accumulate ? *dst + val : val;
            }
        }
    }
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
    int G, H, kp, stages, cols, kwc, pitch;
    bool tma;
};

// About one CTA per SM, one warp per (16-row group, K-part); the widest K chunk
// (and up to two columns) whose digit planes fit in shared memory.
Plan make_plan(int out, int kw, int batch) {
    const int sms = num_sms();
    const int groups = (out + 15) / 16;
    const int kwp = (kw + 15) / 16 * 16;
    Plan pl;
    pl.tma = (kw % 4) == 0;
    pl.G = std::max(1, std::min(kMaxWarps, (groups + sms - 1) / sms));
    for (int nchunks = 1;; ++nchunks) {
        pl.kwc = ((kwp + nchunks - 1) / nchunks + 15) / 16 * 16;
        pl.H = std::max(1, std::min(kMaxParts, kMaxWarps / pl.G));
        pl.H = std::min(pl.H, pl.kwc / kStepWords);  // at least one step per part
        pl.kp = ((pl.kwc + pl.H - 1) / pl.H + kStepWords - 1) / kStepWords * kStepWords;
        pl.H = (pl.kwc + pl.kp - 1) / pl.kp;  // drop empty parts
        pl.stages = pl.G * pl.H <= 8 ? 8 : 4;
        pl.pitch = plane_pitch(pl.kwc);
        for (int cols = std::min(kMaxColsPass, batch); cols >= 1; --cols) {
            pl.cols = cols;
            if (gemv_smem(pl.G, pl.H, cols, pl.stages, pl.pitch, pl.tma) <= kSmemBudget) return pl;
        }
    }
}

template <int STAGES, bool TMA>
cudaError_t launch_kernel(const CUtensorMap& map, const GemvArgs& p, cudaStream_t st) {
    const size_t smem = gemv_smem(p.G, p.H, p.ncols, STAGES, p.pitch, TMA);
    static size_t granted[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || granted[dev] < smem) {
        cudaError_t e =
            cudaFuncSetAttribute(gemv_kernel<STAGES, TMA>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
    return cudaLaunchKernelEx(&cfg, gemv_kernel<STAGES, TMA>, map, p);
}

}  // namespace

cudaError_t launch_gemv(const uint32_t* packed, const float* s, int out, int K, const float* u, int batch, float* o,
                        unsigned* status, cudaStream_t st) {
    const int kw = K / 32;
    const Plan pl = make_plan(out, kw, batch);

    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    if (pl.tma) {
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
    for (int c0 = 0; c0 < batch; c0 += pl.cols) {
        for (int kx0 = 0; kx0 < kw; kx0 += pl.kwc) {
            GemvArgs p;
            p.packed = packed;
            p.s = s;
            p.u = u;
            p.o = o;
            p.status = status;
            p.out = out;
            p.K = K;
            p.kw = kw;
            p.c0 = c0;
            p.ncols = std::min(pl.cols, batch - c0);
            p.kx0 = kx0;
            p.kwc = pl.kwc;
            p.G = pl.G;
            p.H = pl.H;
            p.kp = pl.kp;
            p.pitch = pl.pitch;
            p.accumulate = kx0 > 0;
            cudaError_t e = !pl.tma ? launch_kernel<4, false>(map, p, st)
                            : pl.stages == 8 ? launch_kernel<8, true>(map, p, st)
                                             : launch_kernel<4, true>(map, p, st);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaGetLastError();
}

}  // namespace lq
