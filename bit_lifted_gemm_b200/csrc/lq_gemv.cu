// Decode 1-bit GEMV, batch 1..16 (LiftQuant paper note, "Key designs" 4: after
// the small matmul T* a the layer is a 1-bit x float matmul with W_q, then
// diag(s)):
//
//   o[c][r] = s[r] * sum_k sigma[r][k] u[c][k],   sigma = +1 if the bit is set.
//
// Design (integer tensor-core operands, exact accumulation):
//   * sum_k sigma u = 2 sum_{bit=1} u - sum_k u, so only the set bits matter.
//   * Each column of u (over the K range of a launch) becomes 24-bit fixed
//     point with one power-of-two scale (|u_q| < 2^22: an element's rounding
//     error is at most 2^-22 of the column's largest |u|), held as three
//     balanced int8 digit planes u_q = d0 + 2^8 d1 + 2^16 d2 -- the bytes of
//     (u_q + 0x808080) ^ 0x808080. Every CTA quantizes u for itself in its
//     prologue, one 32-element word per thread: each warp brings its words into
//     shared memory with TMA (128-byte swizzle, so the per-thread reads are
//     conflict-free) ahead of its remaining weight prefetch; no workspace, no
//     extra launch.
//   * A sign word w yields eight u8 operand registers w & (0x01010101 << j),
//     j = 0..7: bytes 0 or 2^j for bits j, j+8, j+16, j+24 -- one LOP3 per four
//     weights, nothing unpacked to memory. These are the A fragments of
//     mma.sync m16n8k32 u8 x s8 -> s32. (Measured on B200: 0.5 such MMA per
//     clock per SM = 256 weight bits/clk/SM in isolation, against ~186 weight
//     bits/clk/SM that saturate HBM at 1.97 GHz; the LOP3s load the integer
//     ALU at the same rate, so the step body carries as little else as
//     possible. tcgen05 kind::i8 with N <= 64 sustains one MMA per ~46 clocks
//     = 90 bits/clk/SM, and e4m3 mma.sync runs ~2.6x slower than u8 in this
//     loop: both too slow at decode batch sizes.) B fragments are the digit
//     planes (MMA column n = 3c + p), read from shared memory where word pair
//     (x, x+1), x even, sits in the four 16-byte chunks from 2x + x/4 (a bank
//     skew), chunk r holding (2r, x), (2r, x+1), (2r+1, x), (2r+1, x+1), so one
//     conflict-free 16-byte load yields the (adjacent) B register pairs of two
//     j. One s32 accumulator set per j keeps the 2^j scales apart; every
//     integer sum is exact.
//   * One CTA of 12 warps per SM (three per scheduler). A CTA owns a run of
//     16-row groups; the (group, tile) sequence of its groups is cut into 12
//     equal contiguous ranges, one per warp, so every scheduler carries the
//     same load whatever the shape. A tile is two 16-word steps of 16 rows
//     (2 KB, one 3-D TMA box) when the row length allows, else one step. Each
//     warp streams its tiles through a private ring, one mbarrier per stage,
//     every wait bounded. A warp adds the exact integer total of each group it
//     touches into the CTA's per-(group, column, row) sums with 64-bit shared
//     atomics: integer addition, so the result does not depend on the order.
//   * The GEMV is launched as a programmatic dependent of whatever precedes it
//     on the stream (normally the activation lift): it requests its first
//     weight tiles early and waits (griddepcontrol.wait) only before reading u.
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

constexpr int kWarps = 12;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxColsPass = 2;   // batch columns per pass (6 digit planes <= n8)
constexpr int kStepWords = 16;    // words per row a warp consumes per step
constexpr int kStepBytes = 16 * kStepWords * 4;  // one step of 16 rows x 64 bytes
constexpr int kMaxRounds = 2;     // quantization items per thread kept in registers (staged path)
constexpr int kUBoxRows = 16;     // words per TMA box of u
constexpr int kWordsPerSweep = kThreads / 8;  // direct u path: eight threads per 32-element word
constexpr int kMaxSegSteps = 255;  // steps one 32-bit segment sum holds
constexpr size_t kSmemBudget = 220 * 1024;

// Digit-plane storage: 16-byte chunks; word pair (x, x+1), x even, occupies the
// four chunks from 2x + x/4.
__host__ __device__ __forceinline__ int chunkpos(int x) { return 2 * x + (x >> 2); }

// Chunks per plane for `words` words: covers chunkpos(words - 1) + 4 and is
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

// One 16-word step of one 16-row group: words 4t..4t+3 of rows g (ca) and g+8
// (cb) against this lane's digit chunks bp[0..7].
__device__ __forceinline__ void mma_step(int (&acc)[8][4], const uint4& ca, const uint4& cb, const uint4* bp) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t a0 = h ? ca.z : ca.x, a2 = h ? ca.w : ca.y;  // row g: words 4t+2h, 4t+2h+1
        const uint32_t a1 = h ? cb.z : cb.x, a3 = h ? cb.w : cb.y;  // row g+8
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint4 b = bp[4 * h + r];  // (2r, x) (2r, x+1) (2r+1, x) (2r+1, x+1)
            const uint32_t m = 0x01010101u << (2 * r), n = m << 1;
            mma_u8s8(acc[2 * r], a0 & m, a1 & m, a2 & m, a3 & m, b.x, b.y);
            mma_u8s8(acc[2 * r + 1], a0 & n, a1 & n, a2 & n, a3 & n, b.z, b.w);
        }
    }
}

__device__ __forceinline__ uint4 load_words(const uint32_t* row, int x, int kw) {
    uint4 v;
    v.x = x < kw ? __ldg(row + x) : 0u;
    v.y = x + 1 < kw ? __ldg(row + x + 1) : 0u;
    v.z = x + 2 < kw ? __ldg(row + x + 2) : 0u;
    v.w = x + 3 < kw ? __ldg(row + x + 3) : 0u;
    return v;
}

// floor(i * n / parts) for i <= 256, in 32-bit arithmetic when the product fits.
__device__ __forceinline__ int split_point(unsigned i, unsigned n, unsigned parts) {
    return n < (1u << 24) ? (int)(i * n / parts) : (int)((unsigned long long)i * n / parts);
}

// 2^e as a float for -126 <= e <= 127.
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// Exponent e with cmax < 2^e (frexp convention) from the bits of cmax >= 0;
// zero and subnormal maxima use e = -126.
__device__ __forceinline__ int max_exponent(unsigned cmax_bits) {
    const int E = (cmax_bits >> 23) & 255;
    return E == 0 ? -126 : E - 126;
}

// 32 elements of staged row `row` (128 bytes, 128-byte swizzle: 16-byte chunk q
// of row r sits at chunk q ^ (r & 7)), or zeros when !valid.
__device__ __forceinline__ void read_staged(const uint8_t* stage, int row, bool valid, float (&v)[32]) {
    const uint8_t* base = stage + (size_t)row * 128;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 f = valid ? *reinterpret_cast<const float4*>(base + ((q ^ (row & 7)) << 4))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        v[4 * q] = f.x;
        v[4 * q + 1] = f.y;
        v[4 * q + 2] = f.z;
        v[4 * q + 3] = f.w;
    }
}

// x + 1.5 * 2^23 rounds x to the nearest integer (ties to even) in the low
// mantissa bits when |x| <= 2^22: the integer is then bits - 0x4B400000.
constexpr float kRoundMagic = 12582912.0f;
constexpr uint32_t kMagicBits = 0x4B400000u;

// Digits of one word: P[pl][j] holds, in byte i, digit pl of element j + 8 i.
// Returns sum_e u_q[e] (|sum| < 2^27).
// ONE: the scale is the single float sa (column maxima above 2^-104; one
// rounding multiply-add per element); else sa * sb in two exact steps.
template <bool ONE>
__device__ __forceinline__ int word_digits(const float (&v)[32], float sa, float sb, uint32_t (&P)[3][8]) {
    uint32_t tb[32];  // balanced digits of element e in bytes 0..2 of tb[e]
    uint32_t bsum = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const uint32_t b = __float_as_uint(ONE ? fmaf(v[e], sa, kRoundMagic)
                                               : fmaf(v[e] * sa, sb, kRoundMagic));  // u_q = b - kMagicBits
        bsum += b;
        tb[e] = (b - (kMagicBits - 0x808080u)) ^ 0x808080u;  // (u_q + 0x808080) ^ 0x808080
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // 4x3 byte transpose of elements j, j+8, j+16, j+24
        const uint32_t t0 = __byte_perm(tb[j], tb[j + 8], 0x5140);        // a0 b0 a1 b1
        const uint32_t t1 = __byte_perm(tb[j + 16], tb[j + 24], 0x5140);  // c0 d0 c1 d1
        const uint32_t t2 = __byte_perm(tb[j], tb[j + 8], 0x0062);        // a2 b2 .  .
        const uint32_t t3 = __byte_perm(tb[j + 16], tb[j + 24], 0x0062);  // c2 d2 .  .
        P[0][j] = __byte_perm(t0, t1, 0x5410);
        P[1][j] = __byte_perm(t0, t1, 0x7632);
        P[2][j] = __byte_perm(t2, t3, 0x5410);
    }
    return (int)(bsum - 32u * kMagicBits);
}

// Elements j, j + 8, j + 16, j + 24 of word x of a column of u (zeros past the
// end of K): the four bytes of one B register.
__device__ __forceinline__ float4 load_quarter(const float* uc, int x, int kw, int j) {
    if (x >= kw) return make_float4(0.f, 0.f, 0.f, 0.f);
    const float* q = uc + 32 * x + j;
    return make_float4(__ldg(q), __ldg(q + 8), __ldg(q + 16), __ldg(q + 24));
}

// Digits of four elements (j, j + 8, j + 16, j + 24 of a word): plane pl of
// P[pl] in bytes 0..3. Returns their sum of u_q.
__device__ __forceinline__ int quarter_digits(const float4& v, float sa, float sb, uint32_t (&P)[3]) {
    const float e[4] = {v.x, v.y, v.z, v.w};
    uint32_t tb[4];
    uint32_t bsum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t b = __float_as_uint(fmaf(e[i] * sa, sb, kRoundMagic));  // u_q = b - kMagicBits
        bsum += b;
        tb[i] = (b - (kMagicBits - 0x808080u)) ^ 0x808080u;  // (u_q + 0x808080) ^ 0x808080
    }
    const uint32_t t0 = __byte_perm(tb[0], tb[1], 0x5140);  // a0 b0 a1 b1
    const uint32_t t1 = __byte_perm(tb[2], tb[3], 0x5140);  // c0 d0 c1 d1
    const uint32_t t2 = __byte_perm(tb[0], tb[1], 0x0062);  // a2 b2 .  .
    const uint32_t t3 = __byte_perm(tb[2], tb[3], 0x0062);  // c2 d2 .  .
    P[0] = __byte_perm(t0, t1, 0x5410);
    P[1] = __byte_perm(t0, t1, 0x7632);
    P[2] = __byte_perm(t2, t3, 0x5410);
    return (int)(bsum - 4u * kMagicBits);
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
    int ngroups;      // 16-row groups of the layer; CTA b owns [b*ngroups/grid, (b+1)*ngroups/grid)
    int maxgroups;    // most 16-row groups a CTA owns
    int pitch;        // chunks per shared-memory digit plane
    int accumulate;   // 1: o += this launch's result
};

// Shared-memory carve-up (offsets from a 1024-byte-aligned base).
struct Layout {
    size_t ring, work, zero, bars, gacc, sall, colmax, srow, total;
};

__host__ __device__ inline Layout gemv_layout(int ts, int stages, bool tma, bool ustage, int ncols, int kwc,
                                              int pitch, int maxgroups) {
    Layout L;
    L.ring = 0;
    const size_t rings = tma ? (size_t)kWarps * stages * ts * kStepBytes : 0;
    L.work = rings;  // staged u (until quantized), then the digit planes
    const size_t planes = (size_t)3 * ncols * pitch * 16;
    const size_t staged = ustage ? (size_t)ncols * kwc * 128 : 0;
    L.zero = L.work + (((planes > staged ? planes : staged) + 127) & ~(size_t)127);
    L.bars = L.zero + 128;
    L.gacc = L.bars + (size_t)kWarps * (stages + 1) * 8;
    L.sall = L.gacc + (size_t)maxgroups * ncols * 16 * 8;
    L.colmax = L.sall + kMaxColsPass * 8;
    L.srow = L.colmax + kMaxColsPass * 4;
    L.total = L.srow + (size_t)kThreads * 4 + 1024;  // + alignment slack
    return L;
}

// Digits of word xl of column c into the shared planes: chunk r of the pair
// holds 32-bit words (2r, x), (2r, x+1), (2r+1, x), (2r+1, x+1).
__device__ __forceinline__ void store_digits(uint4* planes, int pitch, int c, int xl, const uint32_t (&P)[3][8]) {
    uint32_t* base = reinterpret_cast<uint32_t*>(planes + chunkpos(xl & ~1)) + (xl & 1);
#pragma unroll
    for (int pl = 0; pl < 3; ++pl) {
        uint32_t* d = base + (size_t)(3 * c + pl) * pitch * 4;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            d[4 * r] = P[pl][2 * r];
            d[4 * r + 2] = P[pl][2 * r + 1];
        }
    }
}

// Per-column max of |u| (as float bits) into colmax: one shared atomic per warp
// when the warp's items share a column.
__device__ __forceinline__ void reduce_max(unsigned* colmax, bool live, int c, unsigned bits, int lane) {
    const int c_first = __shfl_sync(0xffffffffu, c, 0);
    if (__all_sync(0xffffffffu, !live || c == c_first)) {
        const unsigned m = __reduce_max_sync(0xffffffffu, bits);
        if (lane == 0) atomicMax(colmax + c_first, m);
    } else if (live) {
        atomicMax(colmax + c, bits);
    }
}

// Per-column sum of u_q (|item sum| < 2^27): split into 16-bit halves so the
// 32-bit warp reductions cannot overflow.
__device__ __forceinline__ void reduce_sum(unsigned long long* sall, bool live, int c, int qsum, int lane) {
    const int c_first = __shfl_sync(0xffffffffu, c, 0);
    if (__all_sync(0xffffffffu, !live || c == c_first)) {
        const unsigned lo = __reduce_add_sync(0xffffffffu, (unsigned)(qsum & 0xffff));
        const int hi = (int)__reduce_add_sync(0xffffffffu, (unsigned)(qsum >> 16));
        if (lane == 0) atomicAdd(sall + c_first, (unsigned long long)(((long long)hi << 16) + (long long)lo));
    } else if (live) {
        atomicAdd(sall + c, (unsigned long long)(long long)qsum);
    }
}

__device__ __forceinline__ float absmax32(const float (&v)[32]) {
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fabsf(v[e]));
    return mx;
}

// TS: steps per ring tile (2 with the 3-D weight map, else 1); STAGES: ring
// depth; TMA: weights through the rings (else guarded register loads); USTAGE:
// u staged in shared memory by TMA (at most kMaxRounds items per thread).
template <int TS, int STAGES, bool TMA, bool USTAGE>
__global__ void __maxnreg__(128)  // 384 threads: leaves registers for the lift beside it
    gemv_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap umap, const GemvArgs p) {
    // a dependent launch (the next K chunk or column pass) may be scheduled as
    // SMs free up; it reads u and o only after its own griddepcontrol.wait,
    // which waits for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned (the 128-byte swizzle of staged u); offsetting the array
    // itself keeps every derived pointer in the shared address space
    uint8_t* smem = smem_raw + ((1024u - (sm100::smem_addr(smem_raw) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int gbeg = split_point(blockIdx.x, p.ngroups, gridDim.x);
    const int gend = split_point(blockIdx.x + 1, p.ngroups, gridDim.x);
    const int m0 = 16 * gbeg;
    const int spg = p.kwc / kStepWords;              // steps per group
    const int tpg = (spg + TS - 1) / TS;             // tiles per group
    const int total = (gend - gbeg) * tpg;           // tiles of this CTA
    const int t0 = split_point(warp, total, kWarps);
    const int t1 = split_point(warp + 1, total, kWarps);
    const int ndig = 3 * p.ncols;
    constexpr int kTileBytes = TS * kStepBytes;

    const Layout L = gemv_layout(TS, STAGES, TMA, USTAGE, p.ncols, p.kwc, p.pitch, p.maxgroups);
    uint8_t* ring = smem + L.ring + (size_t)warp * STAGES * kTileBytes;
    uint8_t* work = smem + L.work;
    uint4* bplanes = reinterpret_cast<uint4*>(work);
    uint4* bzero = reinterpret_cast<uint4*>(smem + L.zero);  // 8 zero chunks: digits of idle MMA columns
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * (STAGES + 1);  // ring stages, then u
    // sum_{bit=1} u_q per (group, column, row), exact integers added with shared
    // atomics (the same result in any order)
    unsigned long long* gacc = reinterpret_cast<unsigned long long*>(smem + L.gacc);
    unsigned long long* sall = reinterpret_cast<unsigned long long*>(smem + L.sall);
    unsigned* colmax = reinterpret_cast<unsigned*>(smem + L.colmax);
    float* srow = reinterpret_cast<float*>(smem + L.srow);  // s of this CTA's first kThreads rows
    const uint32_t ubar = sm100::smem_addr(bars + STAGES);

    // Next tile to request (lane 0): ring index nxt, step xs of its group, row y.
    int nxt = t0, nxt_xs = 0, nxt_y = 0;
    if (TMA) {
        const int gl = t0 / tpg;
        nxt_xs = (t0 - gl * tpg) * TS;
        nxt_y = m0 + 16 * gl;
    }
    auto issue = [&]() {
        const int slot = (nxt - t0) & (STAGES - 1);
        const uint32_t bar = sm100::smem_addr(bars + slot);
        const uint32_t dst = sm100::smem_addr(ring + slot * kTileBytes);
        sm100::mbar_arrive_expect_tx(bar, kTileBytes);
        if (TS == 2)
            sm100::tma_load_3d(dst, &wmap, 0, nxt_y, p.kx0 / kStepWords + nxt_xs, bar);
        else
            sm100::tma_load_2d(dst, &wmap, p.kx0 + nxt_xs * kStepWords, nxt_y, bar);
        ++nxt;
        nxt_xs += TS;
        if (nxt_xs >= spg) {
            nxt_xs = 0;
            nxt_y += 16;
        }
    };
    // One tile (two for shallow rings of 1-step tiles) is requested before the
    // dependency wait, overlapping the kernel before this one; the rest only
    // after this warp's requests for u, so that those latency-critical loads do
    // not queue behind ~100 KB of weights per SM.
    constexpr int kEarly = TS == 1 && STAGES > 4 ? 2 : 1;
    if (lane == 0) {
        if (TMA) sm100::prefetch_tensormap(&wmap);
        if (USTAGE) sm100::prefetch_tensormap(&umap);
        if (TMA || USTAGE) {
            for (int st = 0; st <= STAGES; ++st) sm100::mbar_init(sm100::smem_addr(bars + st), 1);
            sm100::fence_barrier_init();
        }
        if (TMA)
            while (nxt < t1 && nxt < t0 + kEarly) issue();
    }
    if (threadIdx.x < 8) bzero[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x < kMaxColsPass) {
        colmax[threadIdx.x] = 0u;
        sall[threadIdx.x] = 0ull;
    }
    for (int i = threadIdx.x; i < (gend - gbeg) * p.ncols * 16; i += kThreads) gacc[i] = 0ull;
    // s of this CTA's rows is a weight: requested now, stored to shared memory
    // only before the first barrier of the quantization (its latency hides
    // behind the dependency wait and the landing of u)
    const int nrow = (gend - gbeg) * 16;
    const float s_own = threadIdx.x < nrow && m0 + threadIdx.x < p.out ? __ldg(p.s + m0 + threadIdx.x) : 0.f;
    __syncthreads();

    // u is written by the kernel before this one on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- quantize this launch's slice of u: item it = (column, word), item
    // rd * kThreads + threadIdx.x in round rd; pass 1 takes the per-column
    // maxima, pass 2 writes the digit planes
    const int nitems = p.ncols * p.kwc;
    const int nrounds = (nitems + kThreads - 1) / kThreads;
    const int jq = threadIdx.x & 7, wq = threadIdx.x >> 3;  // direct path: element group, word of the sweep
    float v[kMaxRounds][32];
    bool ufail = false;
    if constexpr (USTAGE) {
        // this warp's items of every round, 16 words per box, staged at row = item
        if (lane == 0) {
            uint32_t bytes = 0;
            for (int rd = 0; rd < nrounds; ++rd)
                for (int h = 0; h < 2; ++h)
                    if (rd * kThreads + 32 * warp + kUBoxRows * h < nitems) bytes += kUBoxRows * 128;
            if (bytes) {
                sm100::mbar_arrive_expect_tx(ubar, bytes);
                for (int rd = 0; rd < nrounds; ++rd)
                    for (int h = 0; h < 2; ++h) {
                        const int base = rd * kThreads + 32 * warp + kUBoxRows * h;
                        if (base >= nitems) continue;
                        const int c = base / p.kwc;
                        sm100::tma_load_2d(sm100::smem_addr(work + (size_t)base * 128), &umap, 0,
                                           (p.c0 + c) * p.kw + p.kx0 + (base - c * p.kwc), ubar);
                    }
            } else {
                sm100::mbar_arrive(ubar);
            }
            if (TMA)
                while (nxt < t1 && nxt < t0 + STAGES - 1) issue();
        }
        ufail = !sm100::mbar_wait(ubar, 0, p.status);
#pragma unroll
        for (int rd = 0; rd < kMaxRounds; ++rd) {
            if (rd < nrounds) {
                const int it = rd * kThreads + threadIdx.x;
                const bool live = it < nitems;
                const int c = live ? it / p.kwc : 0;
                read_staged(work, it, live && p.kx0 + it - c * p.kwc < p.kw, v[rd]);
                reduce_max(colmax, live, c, __float_as_uint(absmax32(v[rd])), lane);
            }
        }
    } else {
        // u read directly, eight threads per word: thread jq of a word takes its
        // elements jq, jq + 8, jq + 16, jq + 24. A warp's four words never cross a
        // column (K chunks are multiples of 16 words). Four sweeps of 48 words
        // are in flight at once.
        if (TMA && lane == 0)
            while (nxt < t1 && nxt < t0 + STAGES - 1) issue();
        for (int w0 = 0; w0 < nitems; w0 += 4 * kWordsPerSweep) {
            float4 q[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int it = w0 + k * kWordsPerSweep + wq;
                const int c = it < nitems ? it / p.kwc : 0;
                q[k] = load_quarter(p.u + (long long)(p.c0 + c) * p.K, it < nitems ? p.kx0 + it - c * p.kwc : p.kw,
                                    p.kw, jq);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int it = w0 + k * kWordsPerSweep + wq;
                const bool live = it < nitems;
                const float mx = fmaxf(fmaxf(fabsf(q[k].x), fabsf(q[k].y)), fmaxf(fabsf(q[k].z), fabsf(q[k].w)));
                reduce_max(colmax, live, live ? it / p.kwc : 0, __float_as_uint(mx), lane);
            }
        }
    }
    if (threadIdx.x < nrow) srow[threadIdx.x] = s_own;
    __syncthreads();  // every staged word has been read: the planes may overwrite the staging area
    if constexpr (USTAGE) {
#pragma unroll
        for (int rd = 0; rd < kMaxRounds; ++rd) {
            if (rd >= nrounds) break;
            const int it = rd * kThreads + threadIdx.x;
            const bool live = it < nitems;
            const int c = live ? it / p.kwc : 0;
            const int xl = it - c * p.kwc;
            int qsum = 0;
            if (live) {
                const int F = 22 - max_exponent(colmax[c]);  // column max * 2^F < 2^22
                uint32_t P[3][8];
                // 2^F as one factor when it is a float, else as two exact halves
                if (F <= 127)
                    qsum = word_digits<true>(v[rd], pow2f(F), 1.0f, P);
                else
                    qsum = word_digits<false>(v[rd], pow2f(F >> 1), pow2f(F - (F >> 1)), P);
                store_digits(bplanes, p.pitch, c, xl, P);
            }
            reduce_sum(sall, live, c, qsum, lane);
        }
    } else {
        for (int w0 = 0; w0 < nitems; w0 += 4 * kWordsPerSweep) {
            float4 q[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int it = w0 + k * kWordsPerSweep + wq;
                const int c = it < nitems ? it / p.kwc : 0;
                q[k] = load_quarter(p.u + (long long)(p.c0 + c) * p.K, it < nitems ? p.kx0 + it - c * p.kwc : p.kw,
                                    p.kw, jq);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int it = w0 + k * kWordsPerSweep + wq;
                const bool live = it < nitems;
                const int c = live ? it / p.kwc : 0;
                int qsum = 0;
                if (live) {
                    const int xl = it - c * p.kwc;
                    const int F = 22 - max_exponent(colmax[c]);
                    uint32_t P[3];
                    qsum = quarter_digits(q[k], pow2f(F >> 1), pow2f(F - (F >> 1)), P);
                    // element jq of word pair (xl & ~1): word 2 (jq >> 1) + (jq & 1) of its chunk run
                    uint32_t* base = reinterpret_cast<uint32_t*>(bplanes + chunkpos(xl & ~1)) + (xl & 1) +
                                     4 * (jq >> 1) + 2 * (jq & 1);
#pragma unroll
                    for (int pl = 0; pl < 3; ++pl) base[(size_t)(3 * c + pl) * p.pitch * 4] = P[pl];
                }
                reduce_sum(sall, live, c, qsum, lane);
            }
        }
    }
    __syncthreads();

    // ---- main loop: this warp's tiles [t0, t1), one segment per group touched
    const bool live_col = g < ndig;
    const uint4* bcol = live_col ? bplanes + (size_t)g * p.pitch + 9 * t : bzero;
    const int binc = live_col ? 36 : 0;  // chunkpos advances 36 chunks per 16-word step
    const uint8_t* ring_lane = ring + g * 64 + t * 16;
    const uint32_t bar0 = sm100::smem_addr(bars);
    const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
    int kfail = -1;  // ring index whose wait ran out
    for (int tt = t0; tt < t1;) {
        const int gl = tt / tpg;
        const int tend = min(t1, (gl + 1) * tpg);
        int acc[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = 0;
        int xs = (tt - gl * tpg) * TS;
        const uint4* bp = bcol + binc * xs;
        const int r0 = m0 + 16 * gl + g, r1 = r0 + 8;
        const uint32_t* row0 = p.packed + (long long)min(r0, p.out - 1) * p.kw;
        const uint32_t* row1 = p.packed + (long long)min(r1, p.out - 1) * p.kw;
        const bool v0 = r0 < p.out, v1 = r1 < p.out;
        for (; tt < tend; ++tt, xs += TS) {
            uint4 ca0, cb0, ca1 = zero4, cb1 = zero4;
            if (TMA) {
                const int k = tt - t0;
                const uint32_t bar = bar0 + 8 * (k & (STAGES - 1));
                const uint32_t par = (k / STAGES) & 1;
                if (!sm100::mbar_try_wait(bar, par) && !sm100::mbar_wait(bar, par, p.status)) {
                    kfail = k;  // flagged in the status word; results invalid
                    break;
                }
                const uint8_t* st = ring_lane + (k & (STAGES - 1)) * kTileBytes;
                ca0 = *reinterpret_cast<const uint4*>(st);
                cb0 = *reinterpret_cast<const uint4*>(st + 8 * 64);
                if (TS == 2) {
                    ca1 = *reinterpret_cast<const uint4*>(st + kStepBytes);
                    cb1 = *reinterpret_cast<const uint4*>(st + kStepBytes + 8 * 64);
                }
                __syncwarp();  // every lane has read the slot before lane 0 refills the previous one
                if (lane == 0 && nxt < t1) issue();
            } else {
                const int x = p.kx0 + xs * kStepWords + 4 * t;
                ca0 = v0 ? load_words(row0, x, p.kw) : zero4;
                cb0 = v1 ? load_words(row1, x, p.kw) : zero4;
            }
            mma_step(acc, ca0, cb0, bp);
            bp += binc;
            if (TS == 2) {  // the K chunk of two-step tiles is a multiple of 32 words
                mma_step(acc, ca1, cb1, bp);
                bp += binc;
            }
        }
        if (kfail >= 0) break;
        // ---- segment partial: V = sum_j 2^(7-j) acc_j = 2^7 sum_{bit=1} d per digit
        // column (|V| < 2^23 per step, so 32 bits hold up to 255 steps); the three
        // planes of each batch column are gathered with shuffles and sum_{bit=1}
        // u_q is added into the CTA's per-(group, column, row) total
        int vreg[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int vv = acc[0][e];
#pragma unroll
            for (int j = 1; j < 8; ++j) vv = 2 * vv + acc[j][e];
            vreg[e] = vv;
        }
        unsigned long long* gdst = gacc + (size_t)gl * p.ncols * 16;
#pragma unroll
        for (int c = 0; c < kMaxColsPass; ++c) {
            if (c >= p.ncols) break;
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {  // rows g (hr = 0) and g + 8
                long long s1 = 0;
#pragma unroll
                for (int pl = 0; pl < 3; ++pl) {
                    const int col = 3 * c + pl;
                    const int vv = __shfl_sync(0xffffffffu, vreg[2 * hr + (col & 1)], (lane & ~3) | (col >> 1));
                    s1 += (long long)vv << (8 * pl);  // exact: 2^7 sum_{bit=1} u_q
                }
                if (t == 0) atomicAdd(gdst + c * 16 + g + 8 * hr, (unsigned long long)(s1 >> 7));
            }
        }
    }
    if (lane == 0) {
        // leave nothing in flight after a wait ran out: wait (bounded) for the
        // tiles requested from the failed one on, and for u
        if (TMA && kfail >= 0)
            for (int k = kfail; k < nxt - t0; ++k)
                sm100::mbar_wait(bar0 + 8 * (k & (STAGES - 1)), (k / STAGES) & 1, p.status, 100000000ull);
        if (USTAGE && ufail) sm100::mbar_wait(ubar, 0, p.status, 100000000ull);
    }
    __syncthreads();

    // ---- per (group, column, row): finish and store
    const int nout = (gend - gbeg) * p.ncols * 16;
    for (int item = threadIdx.x; item < nout; item += kThreads) {
        const int row = item & 15, c = (item >> 4) % p.ncols, gl = (item >> 4) / p.ncols;
        const int m = m0 + 16 * gl + row;
        if (m >= p.out) continue;
        const int F = 22 - max_exponent(colmax[c]);
        // sum_k sigma u_q = 2 sum_{bit=1} u_q - sum_k u_q (exact integers), then undo the 2^F scale
        const long long sig = 2 * (long long)gacc[item] - (long long)sall[c];
        const double val = (double)sig * __longlong_as_double((long long)(1023 - F) << 52);
        float* out = p.o + (long long)(p.c0 + c) * p.out + m;
        const float sr = 16 * gl + row < kThreads ? srow[16 * gl + row] : __ldg(p.s + m);
        const float res = (float)(val * (double)sr);
        *out = p.accumulate ? *out + res : res;
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
    int grid, ts, stages, cols, kwc, pitch, maxgroups;
    bool tma, ustage;
    size_t smem;
};

// One CTA per SM (or per group when there are fewer groups). Preference: up to
// two columns per pass, then a deep ring (three tiles in flight per warp), then
// the widest K chunk whose digit planes fit in shared memory (a second launch
// costs less than a shallow ring: measured), then u staged by TMA.
Plan make_plan(int out, int kw, int batch) {
    const int ngroups = (out + 15) / 16;
    Plan pl;
    pl.tma = (kw % 4) == 0;
    pl.ts = pl.tma && kw % 16 == 0 ? 2 : 1;
    const int q = pl.ts * kStepWords;  // K chunks hold whole tiles (zeros past the row end)
    const int kwp = (kw + q - 1) / q * q;
    pl.grid = std::min(num_sms(), ngroups);
    pl.maxgroups = (ngroups + pl.grid - 1) / pl.grid;
    for (int cols = std::min(kMaxColsPass, batch); cols >= 1; --cols) {
        pl.cols = cols;
        for (int deep = pl.tma ? 1 : 0; deep >= 0; --deep) {
            pl.stages = pl.tma ? (pl.ts == 2 ? 2 : 4) * (deep ? 2 : 1) : 4;  // the register path is built for 4
            for (int nchunks = 1; nchunks <= (deep ? 2 : 1 << 20); ++nchunks) {
                pl.kwc = ((kwp + nchunks - 1) / nchunks + q - 1) / q * q;
                if (pl.kwc > kMaxSegSteps * kStepWords) continue;  // 32-bit segment sums
                pl.pitch = plane_pitch(pl.kwc);
                const int nrounds = (cols * pl.kwc + kThreads - 1) / kThreads;
                for (int us = 1; us >= 0; --us) {
                    pl.ustage = us && pl.tma && nrounds <= kMaxRounds;
                    if (us && !pl.ustage) continue;
                    pl.smem = gemv_layout(pl.ts, pl.stages, pl.tma, pl.ustage, cols, pl.kwc, pl.pitch, pl.maxgroups)
                                  .total;
                    if (pl.smem <= kSmemBudget) return pl;
                }
                if (pl.kwc == q) break;  // narrowest chunk already
            }
        }
    }
    return pl;  // nothing fits: the CTA's row partials (maxgroups) are too many; gemv_supported says so
}

template <int TS, int STAGES, bool TMA, bool USTAGE>
cudaError_t launch_kernel(const CUtensorMap& wmap, const CUtensorMap& umap, const GemvArgs& p, const Plan& pl,
                          cudaStream_t st) {
    auto kern = gemv_kernel<TS, STAGES, TMA, USTAGE>;
    static size_t granted[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || granted[dev] < pl.smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) granted[dev] = pl.smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, wmap, umap, p);
}

cudaError_t launch_planned(const CUtensorMap& wmap, const CUtensorMap& umap, const GemvArgs& p, const Plan& pl,
                           cudaStream_t st) {
    if (!pl.tma) return launch_kernel<1, 4, false, false>(wmap, umap, p, pl, st);
    if (pl.ts == 2) {
        if (pl.stages == 4)
            return pl.ustage ? launch_kernel<2, 4, true, true>(wmap, umap, p, pl, st)
                             : launch_kernel<2, 4, true, false>(wmap, umap, p, pl, st);
        return pl.ustage ? launch_kernel<2, 2, true, true>(wmap, umap, p, pl, st)
                         : launch_kernel<2, 2, true, false>(wmap, umap, p, pl, st);
    }
    if (pl.stages == 8)
        return pl.ustage ? launch_kernel<1, 8, true, true>(wmap, umap, p, pl, st)
                         : launch_kernel<1, 8, true, false>(wmap, umap, p, pl, st);
    return pl.ustage ? launch_kernel<1, 4, true, true>(wmap, umap, p, pl, st)
                     : launch_kernel<1, 4, true, false>(wmap, umap, p, pl, st);
}

}  // namespace

bool gemv_supported(int out, int K, int batch) {
    return make_plan(out, K / 32, batch).smem <= kSmemBudget;
}

cudaError_t launch_gemv(const uint32_t* packed, const float* s, int out, int K, const float* u, int batch, float* o,
                        unsigned* status, cudaStream_t st) {
    const int kw = K / 32;
    const Plan pl = make_plan(out, kw, batch);

    CUtensorMap wmap, umap;
    memset(&wmap, 0, sizeof(wmap));
    memset(&umap, 0, sizeof(umap));
    if (pl.tma || pl.ustage) {
        EncodeTiledFn encode = encode_fn();
        if (!encode) return cudaErrorNotSupported;
        if (pl.ts == 2) {  // [chunk of 16 words][row][word in chunk]: one box = two steps of 16 rows
            cuuint64_t gdim[3] = {(cuuint64_t)kStepWords, (cuuint64_t)out, (cuuint64_t)(kw / kStepWords)};
            cuuint64_t gstride[2] = {(cuuint64_t)kw * 4, (cuuint64_t)kStepWords * 4};
            cuuint32_t box[3] = {kStepWords, 16, 2};
            cuuint32_t estride[3] = {1, 1, 1};
            if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(packed), gdim, gstride, box,
                       estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        } else if (pl.tma) {
            cuuint64_t gdim[2] = {(cuuint64_t)kw, (cuuint64_t)out};
            cuuint64_t gstride[1] = {(cuuint64_t)kw * 4};
            cuuint32_t box[2] = {kStepWords, 16};
            cuuint32_t estride[2] = {1, 1};
            if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(packed), gdim, gstride, box,
                       estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        if (pl.ustage) {  // u as rows of one word (32 floats, 128 bytes)
            cuuint64_t gdim[2] = {32, (cuuint64_t)batch * kw};
            cuuint64_t gstride[1] = {128};
            cuuint32_t box[2] = {32, kUBoxRows};
            cuuint32_t estride[2] = {1, 1};
            if (encode(&umap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(u), gdim, gstride, box, estride,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
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
            p.ngroups = (out + 15) / 16;
            p.maxgroups = pl.maxgroups;
            p.pitch = pl.pitch;
            p.accumulate = kx0 > 0;
            cudaError_t e = launch_planned(wmap, umap, p, pl, st);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_lift_gemv(const void* a, bool a_bf16, int batch, int in, const float* tinv, int tblk,
                             const float* M, int d, int D, const uint32_t* packed, const float* s, int out, int K,
                             float* u, float* o, unsigned* status, cudaStream_t st) {
    cudaError_t e = launch_lift(a, a_bf16, batch, in, tinv, tblk, M, d, D, u, false, K, status, st);
    if (e != cudaSuccess) return e;
    return launch_gemv(packed, s, out, K, u, batch, o, status, st);  // a programmatic dependent of the lift
}

}  // namespace lq
