// Decode 1-bit GEMV, batch 1..16 (LiftQuant paper note, "Key designs" 4: after
// the small matmul T* a the layer is a 1-bit x float matmul with W_q, then
// diag(s)):
//
//   o[c][r] = s[r] * sum_k sigma[r][k] u[c][k],   sigma = +1 if the bit is set.
//
// One to three columns run on the mma.sync kernel of this file (three only
// for layers under 40 MB of packed weights), which
// quantizes u inside each CTA (a CTA contracts the whole K range of its launch,
// so it needs every digit of it anyway; no extra launch, no scratch): each
// column of the launch's K range becomes 32-bit fixed point with one
// power-of-two scale, u_q = round(u * 2^F), |u_q| <= 2^30, held as four
// balanced int8 digit planes (the bytes of (u_q + 0x80808080) ^ 0x80808080).
// More columns run on the tcgen05 kernel of lq_gemv_tc.cu, which reads
// every weight once for all columns, after the quantizer of lq_quant.cu has
// written the block-scaled form of u once per call (lq_decode.h).
//
// The mma.sync kernel (integer tensor-core operands, exact accumulation):
//   * sum_k sigma u_q = 2 sum_{bit=1} u_q - sum_k u_q, so only the set bits matter.
//   * A sign word w yields eight u8 operand registers w & (0x01010101 << j),
//     j = 0..7: bytes 0 or 2^j for bits j, j+8, j+16, j+24 -- one LOP3 per four
//     weights, nothing unpacked to memory. These are the A fragments of
//     mma.sync m16n8k32 u8 x s8 -> s32. (Measured on B200: 0.5 such MMA per
//     clock per SM = 256 weight bits/clk/SM, against ~186 weight bits/clk/SM
//     that saturate HBM at 1.97 GHz; the LOP3s load the integer ALU at the same
//     rate, so the step body carries as little else as possible.) B fragments
//     are the digit planes (MMA column n = 4c + p: four planes of up to two
//     batch columns fill the n8 tile), written by the CTA into shared memory
//     where word pair (x, x+1), x even, sits in the four 16-byte chunks
//     from 2x + x/4 (a bank skew), chunk r holding (2r, x), (2r, x+1),
//     (2r+1, x), (2r+1, x+1), so one conflict-free 16-byte load yields the
//     (adjacent) B register pairs of two j. One s32 accumulator set per j keeps
//     the 2^j scales apart; every integer sum is exact.
//   * One CTA of 12 warps per SM (three per scheduler). A CTA owns a run of
//     16-row groups; the (group, tile) sequence of its groups is cut into 12
//     equal contiguous ranges, one per warp, so every scheduler carries the
//     same load whatever the shape. A tile is two 16-word steps of 16 rows
//     (2 KB, one 3-D TMA box) when the row length allows, else one step. Each
//     warp streams its tiles through a private ring, one mbarrier per stage,
//     every wait bounded. A warp adds the exact integer total of each group it
//     touches into the CTA's per-(group, column, row) sums with 64-bit shared
//     atomics: integer addition, so the result does not depend on the order.
//   * The kernel is a programmatic dependent of the kernel before it (normally
//     the lift): it requests its first weight tiles early and waits
//     (griddepcontrol.wait) only before it reads u.
//   * Columns holding a NaN are written as NaN. Columns holding +-Inf (and no
//     NaN) are contracted on their Inf pattern: u_q = +1 at +Inf, -1 at -Inf,
//     0 elsewhere. For a row, S = sum sigma u_q counts the +Inf terms minus the
//     -Inf terms and n the Inf elements of the launch's K range, so the row's
//     IEEE sum over the range is +Inf (S == n), -Inf (S == -n), NaN (anything
//     else) or, with no Inf in the range, 0; launches over further K chunks add
//     into o, which composes the same way under IEEE addition.
//   * K is covered by one launch when the digit planes fit in shared memory,
//     else by several launches that add into o in stream order. Rows whose word
//     count is not a multiple of 4 (not 16-byte aligned for TMA) use guarded
//     register loads instead of the ring.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "lq_decode.h"
#include "lq_internal.h"
#include "lq_sm100.cuh"

namespace lq {
namespace {

constexpr int kWarps = 12;
constexpr int kThreads = 32 * kWarps;
constexpr int kStepBytes = 16 * kStepWords * 4;  // one step of 16 rows x 64 bytes
constexpr int kMaxSegSteps = 255;                // steps one 32-bit segment sum holds
constexpr size_t kSmemBudget = 220 * 1024;
constexpr int kMaxRounds = 2;  // staged u: words per thread kept in registers between the passes
constexpr int kUBoxRows = 16;  // words per TMA box of u

// 32 elements of staged word `row` (128 bytes, 128-byte swizzle: 16-byte chunk q
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

// u_q of one element in its column's mode; sa * sb = 2^F in two exact factors.
__device__ __forceinline__ int quant_elem(float x, int mode, float sa, float sb) {
    if (mode == kColFinite) return __float2int_rn((x * sa) * sb);
    if (mode == kColInf) return isinf(x) ? (x > 0.f ? 1 : -1) : 0;
    return 0;
}

// Digit registers of elements j, j + 8, j + 16, j + 24 (u_q values q0..q3):
// byte i of P[pl] is balanced digit pl of u_q[j + 8 i] (the bytes of
// (u_q + 0x80808080) ^ 0x80808080).
__device__ __forceinline__ void digit_regs(int q0, int q1, int q2, int q3, uint32_t (&P)[kPlanes]) {
    const uint32_t t0 = ((uint32_t)q0 + 0x80808080u) ^ 0x80808080u;
    const uint32_t t1 = ((uint32_t)q1 + 0x80808080u) ^ 0x80808080u;
    const uint32_t t2 = ((uint32_t)q2 + 0x80808080u) ^ 0x80808080u;
    const uint32_t t3 = ((uint32_t)q3 + 0x80808080u) ^ 0x80808080u;
    const uint32_t a01 = __byte_perm(t0, t1, 0x5140), a23 = __byte_perm(t2, t3, 0x5140);  // bytes 0, 1
    const uint32_t b01 = __byte_perm(t0, t1, 0x7362), b23 = __byte_perm(t2, t3, 0x7362);  // bytes 2, 3
    P[0] = __byte_perm(a01, a23, 0x5410);
    P[1] = __byte_perm(a01, a23, 0x7632);
    P[2] = __byte_perm(b01, b23, 0x5410);
    P[3] = __byte_perm(b01, b23, 0x7632);
}

// Byte offset of digit register (j, xl) within a plane: word pair (x, x+1), x
// even, occupies the four 16-byte chunks from chunkpos(x); chunk r holds
// (2r, x), (2r, x+1), (2r+1, x), (2r+1, x+1).
__device__ __forceinline__ int digit_offset(int j, int xl) {
    return (chunkpos(xl & ~1) + (j >> 1)) * 16 + (2 * (j & 1) + (xl & 1)) * 4;
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

// What the epilogue needs per batch column of a launch.
struct ColInfo {
    long long sall;  // sum of u_q over the launch's K range
    int F, mode, ninf, pad;
};

struct GemvArgs {
    const uint32_t* packed;
    const float* s;
    float* o;          // [batch][out]
    const float* u;    // [batch][K]
    unsigned* status;
    int out, K, kw;
    int c0, ncols;    // columns [c0, c0 + ncols) in this pass (ncols <= 2)
    int kx0, kwc;     // words [kx0, kx0 + kwc) of K in this launch; kx0, kwc multiples of 16
    int ngroups;      // 16-row groups of the layer; CTA b owns [b*ngroups/grid, (b+1)*ngroups/grid)
    int maxgroups;    // most 16-row groups a CTA owns
    int pitch;        // chunks per shared-memory digit plane
    unsigned image_bytes;
    int accumulate;   // 1: o += this launch's result
};

// Shared-memory carve-up (offsets from a 1024-byte-aligned base).
struct Layout {
    size_t ring, work, zero, bars, gacc, cinfo, srow, total;
};

__host__ __device__ inline Layout gemv_layout(int ts, int stages, bool tma, bool ustage, size_t image_bytes,
                                              int ncols, int kwc, int maxgroups) {
    Layout L;
    L.ring = 0;
    const size_t rings = tma ? (size_t)kWarps * stages * ts * kStepBytes : 0;
    L.work = rings;  // staged u (until quantized), then the digit planes
    const size_t staged = ustage ? (size_t)ncols * kwc * 128 : 0;
    L.zero = L.work + (((image_bytes > staged ? image_bytes : staged) + 127) & ~(size_t)127);
    L.bars = L.zero + 128;
    L.gacc = L.bars + (size_t)kWarps * (stages + 1) * 8;
    L.cinfo = L.gacc + (size_t)maxgroups * ncols * 16 * 8;
    L.srow = L.cinfo + kMaxColsPass * sizeof(ColInfo);
    L.total = L.srow + (size_t)kThreads * 4 + 1024;  // + alignment slack
    return L;
}

// TS: steps per ring tile (2 with the 3-D weight map, else 1); STAGES: ring
// depth; TMA: weights through the rings (else guarded register loads).
template <int TS, int STAGES, bool TMA, bool USTAGE>
__global__ void __maxnreg__(128)  // 384 threads: leaves registers for a lift beside it
    gemv_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap umap,
                const GemvArgs p) {
    // a dependent launch (the next K chunk or column pass) may be scheduled as
    // SMs free up; it reads o only after its own griddepcontrol.wait, which
    // waits for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base; offsetting the array itself keeps every derived
    // pointer in the shared address space
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
    const int ndig = kPlanes * p.ncols;
    constexpr int kTileBytes = TS * kStepBytes;

    const Layout L = gemv_layout(TS, STAGES, TMA, USTAGE, p.image_bytes, p.ncols, p.kwc, p.maxgroups);
    uint8_t* ring = smem + L.ring + (size_t)warp * STAGES * kTileBytes;
    uint4* bplanes = reinterpret_cast<uint4*>(smem + L.work);
    uint4* bzero = reinterpret_cast<uint4*>(smem + L.zero);  // 8 zero chunks: digits of idle MMA columns
    // per warp: STAGES ring barriers, then one for its staged words of u
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * (STAGES + 1);
    // sum_{bit=1} u_q per (group, column, row), exact integers added with shared
    // atomics (the same result in any order)
    unsigned long long* gacc = reinterpret_cast<unsigned long long*>(smem + L.gacc);
    ColInfo* cinfo = reinterpret_cast<ColInfo*>(smem + L.cinfo);
    float* srow = reinterpret_cast<float*>(smem + L.srow);  // s of this CTA's first kThreads rows

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
    // after the digit planes have been requested, so that those latency-critical
    // loads do not queue behind ~100 KB of weights per SM.
    constexpr int kEarly = TS == 1 && STAGES > 4 ? 2 : 1;
    __shared__ unsigned s_cmax[kMaxColsPass];            // largest |u| (float bits) per column
    __shared__ unsigned long long s_csum[kMaxColsPass];  // sum of u_q per column (two's complement)
    __shared__ int s_cinf[kMaxColsPass];                 // +-Inf elements per column
    if (lane == 0) {
        if (TMA) sm100::prefetch_tensormap(&wmap);
        if (USTAGE) sm100::prefetch_tensormap(&umap);
        for (int st = 0; st <= STAGES; ++st) sm100::mbar_init(sm100::smem_addr(bars + st), 1);
        sm100::fence_barrier_init();
        if (TMA)
            while (nxt < t1 && nxt < t0 + kEarly) issue();
    }
    if (threadIdx.x < kMaxColsPass) {
        s_cmax[threadIdx.x] = 0u;
        s_csum[threadIdx.x] = 0ull;
        s_cinf[threadIdx.x] = 0;
    }
    if (threadIdx.x < 8) bzero[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < (gend - gbeg) * p.ncols * 16; i += kThreads) gacc[i] = 0ull;
    // s of this CTA's rows is a weight: requested now, stored to shared memory
    // after the dependency wait (its latency hides behind the wait)
    const int nrow = (gend - gbeg) * 16;
    const float s_own = threadIdx.x < nrow && m0 + threadIdx.x < p.out ? __ldg(p.s + m0 + threadIdx.x) : 0.f;
    __syncthreads();

    // u is written by the kernel before this one on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- quantize this launch's slice of u into the digit planes (every CTA for
    // itself: a CTA contracts the whole K range of the launch). Pass 1 takes the
    // largest |u| per column (float bits: NaN > Inf > any finite value), pass 2
    // converts; each thread keeps its maxima, sums and Inf counts per column in
    // registers, reduced once per warp at the end of its pass.
    const int nitems = p.ncols * p.kwc;  // (column, word) items
    unsigned tmax[kMaxColsPass] = {0u, 0u};
    long long tsum[kMaxColsPass] = {0, 0};
    int tinf[kMaxColsPass] = {0, 0};
    auto absmax4 = [](float a, float b, float c, float d) {
        return max(max(__float_as_uint(a) & 0x7fffffffu, __float_as_uint(b) & 0x7fffffffu),
                   max(__float_as_uint(c) & 0x7fffffffu, __float_as_uint(d) & 0x7fffffffu));
    };
    auto add_col = [&](int c, unsigned mx) {
        if (c == 0)
            tmax[0] = max(tmax[0], mx);
        else
            tmax[kMaxColsPass - 1] = max(tmax[kMaxColsPass - 1], mx);
    };
    auto add_sum = [&](int c, long long qs, int ni) {
        if (c == 0) {
            tsum[0] += qs;
            tinf[0] += ni;
        } else {
            tsum[kMaxColsPass - 1] += qs;
            tinf[kMaxColsPass - 1] += ni;
        }
    };
    auto reduce_max = [&]() {
#pragma unroll
        for (int c = 0; c < kMaxColsPass; ++c) {
            const unsigned m = __reduce_max_sync(0xffffffffu, tmax[c]);
            if (lane == 0 && c < p.ncols && m) atomicMax(&s_cmax[c], m);
        }
    };
    int cmode[kMaxColsPass], cF[kMaxColsPass];
    float csa[kMaxColsPass], csb[kMaxColsPass];
    auto column_scales = [&]() {
#pragma unroll
        for (int c = 0; c < kMaxColsPass; ++c) {
            // mode; u_q = round(u * 2^F) with the column maximum below 2^e, F = 30 - e
            // (|u_q| <= 2^30), 2^F as two float factors when it leaves the float range
            const unsigned cm = s_cmax[c];
            cmode[c] = cm > 0x7f800000u ? kColNaN : cm == 0x7f800000u ? kColInf : kColFinite;
            const int E = (int)(cm >> 23);
            cF[c] = cmode[c] == kColFinite ? 30 - (E == 0 ? -126 : E - 126) : 0;
            const int Fa = cF[c] > 127 ? cF[c] / 2 : cF[c];
            csa[c] = __int_as_float((127 + Fa) << 23);
            csb[c] = __int_as_float((127 + cF[c] - Fa) << 23);
        }
    };
    uint8_t* planes8 = reinterpret_cast<uint8_t*>(bplanes);
    bool ufail = false;
    if constexpr (USTAGE) {
        // One word per thread and round: this warp's 32 words of every round come
        // in boxes of 16 (a box never crosses a column: kwc and the item bases are
        // multiples of 16), staged at row = item with the 128-byte swizzle.
        uint8_t* stage = smem + L.work;
        const int nrounds = (nitems + kThreads - 1) / kThreads;
        const uint32_t ubar = sm100::smem_addr(bars + STAGES);
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
                        sm100::tma_load_2d(sm100::smem_addr(stage + (size_t)base * 128), &umap, 0,
                                           (p.c0 + c) * p.kw + p.kx0 + (base - c * p.kwc), ubar);
                    }
            } else {
                sm100::mbar_arrive(ubar);
            }
            // the rest of the weight ring only now: u is on the critical path and
            // must not queue behind ~100 KB of weights per SM
            if (TMA)
                while (nxt < t1 && nxt < t0 + STAGES) issue();
        }
        ufail = !sm100::mbar_wait(ubar, 0, p.status);
        float v[kMaxRounds][32];
#pragma unroll
        for (int rd = 0; rd < kMaxRounds; ++rd) {
            if (rd < nrounds) {
                const int it = rd * kThreads + threadIdx.x;
                const bool live = it < nitems;
                const int c = live ? it / p.kwc : 0;
                read_staged(stage, it, live && !ufail && p.kx0 + it - c * p.kwc < p.kw, v[rd]);
                unsigned mx = 0u;
#pragma unroll
                for (int e = 0; e < 32; e += 4) mx = max(mx, absmax4(v[rd][e], v[rd][e + 1], v[rd][e + 2], v[rd][e + 3]));
                add_col(c, mx);
            }
        }
        reduce_max();
        if (threadIdx.x < nrow) srow[threadIdx.x] = s_own;
        __syncthreads();  // every staged word has been read: the planes may overwrite the staging area
        column_scales();
#pragma unroll
        for (int rd = 0; rd < kMaxRounds; ++rd) {
            if (rd >= nrounds) break;
            const int it = rd * kThreads + threadIdx.x;
            if (it >= nitems) continue;
            const int c = it / p.kwc, xl = it - c * p.kwc;
            const int mode = c == 0 ? cmode[0] : cmode[kMaxColsPass - 1];
            const float sa = c == 0 ? csa[0] : csa[kMaxColsPass - 1], sb = c == 0 ? csb[0] : csb[kMaxColsPass - 1];
            uint8_t* pc = planes8 + (size_t)(kPlanes * c) * p.pitch * 16;
            const size_t pstride = (size_t)p.pitch * 16;
            long long qs = 0;
            int ni = 0;
            if (mode == kColFinite) {  // the common case, without per-element mode tests
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int q0 = __float2int_rn((v[rd][j] * sa) * sb);
                    const int q1 = __float2int_rn((v[rd][j + 8] * sa) * sb);
                    const int q2 = __float2int_rn((v[rd][j + 16] * sa) * sb);
                    const int q3 = __float2int_rn((v[rd][j + 24] * sa) * sb);
                    uint32_t P[kPlanes];
                    digit_regs(q0, q1, q2, q3, P);
                    const int off = digit_offset(j, xl);
#pragma unroll
                    for (int pl = 0; pl < kPlanes; ++pl) *reinterpret_cast<uint32_t*>(pc + pl * pstride + off) = P[pl];
                    // |q0 + q1| <= 2^31 fits unsigned 32-bit arithmetic exactly as a signed 33-bit value
                    qs += (long long)(q0 + (long long)q1) + (long long)(q2 + (long long)q3);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int q0 = quant_elem(v[rd][j], mode, sa, sb), q1 = quant_elem(v[rd][j + 8], mode, sa, sb);
                    const int q2 = quant_elem(v[rd][j + 16], mode, sa, sb);
                    const int q3 = quant_elem(v[rd][j + 24], mode, sa, sb);
                    uint32_t P[kPlanes];
                    digit_regs(q0, q1, q2, q3, P);
                    const int off = digit_offset(j, xl);
#pragma unroll
                    for (int pl = 0; pl < kPlanes; ++pl) *reinterpret_cast<uint32_t*>(pc + pl * pstride + off) = P[pl];
                    qs += (long long)q0 + q1 + q2 + q3;
                    ni += (int)isinf(v[rd][j]) + (int)isinf(v[rd][j + 8]) + (int)isinf(v[rd][j + 16]) +
                          (int)isinf(v[rd][j + 24]);
                }
            }
            add_sum(c, qs, ni);
        }
    } else {
        // u read directly: item (column, word) taken by eight threads; thread jq
        // holds elements jq, jq + 8, jq + 16, jq + 24 of the word, which become
        // the digit register (jq, word) of each plane. A warp's four words lie in
        // one column (kwc is a multiple of 16).
        constexpr int kSweep = kThreads / 8;  // words per sweep
        constexpr int kCached = 8;            // sweeps kept in registers between the passes
        const int jq = threadIdx.x & 7, wq = threadIdx.x >> 3;
        auto load_item = [&](int it) -> float4 {
            const int c = it / p.kwc;
            const int x = p.kx0 + it - c * p.kwc;
            if (it >= nitems || x >= p.kw) return make_float4(0.f, 0.f, 0.f, 0.f);
            const float* q = p.u + (long long)(p.c0 + c) * p.K + 32 * x + jq;
            return make_float4(__ldg(q), __ldg(q + 8), __ldg(q + 16), __ldg(q + 24));
        };
        float4 cache[kCached];
#pragma unroll
        for (int sw = 0; sw < kCached; ++sw)
            if (sw * kSweep < nitems) cache[sw] = load_item(sw * kSweep + wq);  // block-uniform condition
        // the rest of the weight ring only now (after the u requests)
        if (TMA && lane == 0)
            while (nxt < t1 && nxt < t0 + STAGES) issue();
        auto item = [&](int w0) -> float4 {
            const int sw = w0 / kSweep;
            if (sw >= kCached) return load_item(w0 + wq);
            float4 v = cache[0];
#pragma unroll
            for (int k = 1; k < kCached; ++k)
                if (sw == k) v = cache[k];
            return v;
        };
        for (int w0 = 0; w0 < nitems; w0 += kSweep) {
            const float4 v = item(w0);
            add_col(min((w0 + 4 * warp) / p.kwc, kMaxColsPass - 1), absmax4(v.x, v.y, v.z, v.w));  // warp-uniform
        }
        reduce_max();
        if (threadIdx.x < nrow) srow[threadIdx.x] = s_own;
        __syncthreads();
        column_scales();
        for (int w0 = 0; w0 < nitems; w0 += kSweep) {
            const float4 v = item(w0);
            const int it = w0 + wq;
            if (it >= nitems) continue;
            const int c = it / p.kwc, xl = it - c * p.kwc;
            const int mode = c == 0 ? cmode[0] : cmode[kMaxColsPass - 1];
            const float sa = c == 0 ? csa[0] : csa[kMaxColsPass - 1], sb = c == 0 ? csb[0] : csb[kMaxColsPass - 1];
            const int q0 = quant_elem(v.x, mode, sa, sb), q1 = quant_elem(v.y, mode, sa, sb);
            const int q2 = quant_elem(v.z, mode, sa, sb), q3 = quant_elem(v.w, mode, sa, sb);
            uint32_t P[kPlanes];
            digit_regs(q0, q1, q2, q3, P);
            uint8_t* pc = planes8 + (size_t)(kPlanes * c) * p.pitch * 16 + digit_offset(jq, xl);
#pragma unroll
            for (int pl = 0; pl < kPlanes; ++pl) *reinterpret_cast<uint32_t*>(pc + (size_t)pl * p.pitch * 16) = P[pl];
            add_sum(c, (long long)q0 + q1 + q2 + q3,
                    (int)isinf(v.x) + (int)isinf(v.y) + (int)isinf(v.z) + (int)isinf(v.w));
        }
    }
    // per warp and column: |sum| < 2^41 per thread (at most 2^11 elements of
    // |u_q| <= 2^30 each per launch and thread); reduced as the low 16 bits and
    // the rest
#pragma unroll
    for (int c = 0; c < kMaxColsPass; ++c) {
        const unsigned lo = __reduce_add_sync(0xffffffffu, (unsigned)(tsum[c] & 0xffff));
        const long long hiv = tsum[c] >> 16;
        const unsigned hlo = __reduce_add_sync(0xffffffffu, (unsigned)(hiv & 0xffff));
        const int hhi = __reduce_add_sync(0xffffffffu, (int)(hiv >> 16));
        const int ni = __reduce_add_sync(0xffffffffu, tinf[c]);
        if (lane == 0 && c < p.ncols) {
            const long long tot = (long long)lo + ((long long)hlo << 16) + ((long long)hhi << 32);
            atomicAdd(&s_csum[c], (unsigned long long)tot);
            if (ni) atomicAdd(&s_cinf[c], ni);
        }
    }
    __syncthreads();
    if (threadIdx.x < p.ncols) {
        const int c = threadIdx.x;
        ColInfo ci;
        ci.sall = (long long)s_csum[c];
        ci.F = cF[c];
        ci.mode = cmode[c];
        ci.ninf = s_cinf[c];
        ci.pad = 0;
        cinfo[c] = ci;
    }
    __syncthreads();
    const bool pfail = ufail;  // results invalid (flagged in the status word) if u never arrived

    // ---- main loop: this warp's tiles [t0, t1), one segment per group touched
    const bool live_col = g < ndig;
    const uint4* bcol = live_col ? bplanes + (size_t)g * p.pitch + 9 * t : bzero;
    const int binc = live_col ? 36 : 0;  // chunkpos advances 36 chunks per 16-word step
    const uint8_t* ring_lane = ring + g * 64 + t * 16;
    const uint32_t bar0 = sm100::smem_addr(bars);
    const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
    int kfail = pfail ? 0 : -1;  // ring index whose wait ran out (all of them without u)
    for (int tt = t0; tt < t1 && kfail < 0;) {
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
        // column (|V| < 2^23 per step, so 32 bits hold up to 255 steps); the four
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
                for (int pl = 0; pl < kPlanes; ++pl) {
                    const int col = kPlanes * c + pl;
                    const int vv = __shfl_sync(0xffffffffu, vreg[2 * hr + (col & 1)], (lane & ~3) | (col >> 1));
                    s1 += (long long)vv << (8 * pl);  // exact: 2^7 sum_{bit=1} u_q
                }
                if (t == 0) atomicAdd(gdst + c * 16 + g + 8 * hr, (unsigned long long)(s1 >> 7));
            }
        }
    }
    if (lane == 0) {
        // leave nothing in flight after a wait ran out: wait (bounded) for the
        // tiles requested from the failed one on, and for this warp's words of u
        if (TMA && kfail >= 0)
            for (int k = kfail; k < nxt - t0; ++k)
                sm100::mbar_wait(bar0 + 8 * (k & (STAGES - 1)), (k / STAGES) & 1, p.status, 100000000ull);
        if (USTAGE && ufail) sm100::mbar_wait(bar0 + 8 * STAGES, 0, p.status, 100000000ull);
    }
    __syncthreads();

    // ---- per (group, column, row): finish and store
    const int nout = (gend - gbeg) * p.ncols * 16;
    for (int item = threadIdx.x; item < nout; item += kThreads) {
        const int row = item & 15, c = (item >> 4) % p.ncols, gl = (item >> 4) / p.ncols;
        const int m = m0 + 16 * gl + row;
        if (m >= p.out) continue;
        const ColInfo ci = cinfo[c];
        // sum_k sigma u_q = 2 sum_{bit=1} u_q - sum_k u_q (exact integers)
        const long long sig = 2 * (long long)gacc[item] - ci.sall;
        const float sr = 16 * gl + row < kThreads ? srow[16 * gl + row] : __ldg(p.s + m);
        float res;
        if (ci.mode == kColFinite) {  // undo the 2^F scale
            const double val = (double)sig * __longlong_as_double((long long)(1023 - ci.F) << 52);
            res = (float)(val * (double)sr);
        } else if (ci.mode == kColInf) {  // the IEEE sum of this range's Inf terms (none: 0)
            const double inf = __longlong_as_double(0x7ff0000000000000ll);
            const double val = ci.ninf == 0 ? 0.0 : sig == ci.ninf ? inf : sig == -ci.ninf ? -inf : __longlong_as_double(0x7ff8000000000000ll);
            res = ci.ninf == 0 ? 0.f : (float)(val * (double)sr);
        } else {
            res = __int_as_float(0x7fc00000);
        }
        float* outp = p.o + (long long)(p.c0 + c) * p.out + m;
        *outp = p.accumulate ? *outp + res : res;
    }
}

// ---------------------------------------------------------------- host side
int num_sms() {
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    if (dev < 64 && sms[dev]) return sms[dev];
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;  // planning without a device (argument checks on a host without a GPU)
    }
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

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// mma.sync plan: one CTA per SM (or per group when there are fewer groups).
// Preference: up to two columns per pass, then a deep ring (three tiles in
// flight per warp), then the widest K chunk whose digit planes fit in shared
// memory (a second launch costs less than a shallow ring: measured).
bool plan_mma(DecodePlan& pl) {
    const int out = pl.out, kw = pl.kw, batch = pl.batch;
    const long long ngroups = ((long long)out + 15) / 16;
    pl.tma = (kw % 4) == 0;
    pl.ts = pl.tma && kw % 16 == 0 ? 2 : 1;
    const int q = pl.ts * kStepWords;  // K chunks hold whole tiles (zeros past the row end)
    const int kwp = (kw + q - 1) / q * q;
    pl.grid = (int)std::min<long long>(num_sms(), ngroups);
    const long long maxgroups = (ngroups + pl.grid - 1) / pl.grid;
    if (maxgroups > (1 << 20)) return false;
    pl.maxgroups = (int)maxgroups;
    for (int cols = std::min(kMaxColsPass, batch); cols >= 1; --cols) {
        pl.cols = cols;
        for (int deep = pl.tma ? 1 : 0; deep >= 0; --deep) {
            pl.stages = pl.tma ? (pl.ts == 2 ? 2 : 4) * (deep ? 2 : 1) : 4;  // the register path is built for 4
            for (int nchunks = 1; nchunks <= (deep ? 2 : 1 << 20); ++nchunks) {
                pl.kwc = ((kwp + nchunks - 1) / nchunks + q - 1) / q * q;
                if (pl.kwc > kMaxSegSteps * kStepWords) continue;  // 32-bit segment sums
                pl.pitch = plane_pitch(pl.kwc);
                pl.image_bytes = (size_t)kPlanes * cols * pl.pitch * 16;
                const int nrounds = (cols * pl.kwc + kThreads - 1) / kThreads;
                for (int us = 1; us >= 0; --us) {  // u staged by TMA when it fits
                    pl.ustage = us && pl.tma && nrounds <= kMaxRounds;
                    if (us && !pl.ustage) continue;
                    pl.smem = gemv_layout(pl.ts, pl.stages, pl.tma, pl.ustage, pl.image_bytes, cols, pl.kwc,
                                          pl.maxgroups).total;
                    if (pl.smem <= kSmemBudget) {
                        pl.nchunk = (kw + pl.kwc - 1) / pl.kwc;
                        pl.npass = (batch + cols - 1) / cols;
                        return true;
                    }
                }
                if (pl.kwc == q) break;  // narrowest chunk already
            }
        }
    }
    return false;  // the CTA's row partials (maxgroups) are too many
}

template <int TS, int STAGES, bool TMA, bool USTAGE>
cudaError_t launch_kernel(const CUtensorMap& wmap, const CUtensorMap& umap, const GemvArgs& p, const DecodePlan& pl,
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

template <bool US>
cudaError_t launch_planned_us(const CUtensorMap& wmap, const CUtensorMap& umap, const GemvArgs& p,
                              const DecodePlan& pl, cudaStream_t st) {
    if (pl.ts == 2)
        return pl.stages == 4 ? launch_kernel<2, 4, true, US>(wmap, umap, p, pl, st)
                              : launch_kernel<2, 2, true, US>(wmap, umap, p, pl, st);
    return pl.stages == 8 ? launch_kernel<1, 8, true, US>(wmap, umap, p, pl, st)
                          : launch_kernel<1, 4, true, US>(wmap, umap, p, pl, st);
}

cudaError_t launch_planned(const CUtensorMap& wmap, const CUtensorMap& umap, bool ustage, const GemvArgs& p,
                           const DecodePlan& pl, cudaStream_t st) {
    if (!pl.tma) return launch_kernel<1, 4, false, false>(wmap, umap, p, pl, st);
    return ustage ? launch_planned_us<true>(wmap, umap, p, pl, st) : launch_planned_us<false>(wmap, umap, p, pl, st);
}

cudaError_t launch_mma(const uint32_t* packed, const float* s, const DecodePlan& pl, const float* u, float* o,
                       unsigned* status, cudaStream_t st) {
    const int out = pl.out, kw = pl.kw;
    CUtensorMap wmap, umap;
    memset(&wmap, 0, sizeof(wmap));
    memset(&umap, 0, sizeof(umap));
    // u staged by TMA as rows of one 32-element word (128 bytes, 128-byte
    // swizzle) when the plan has room for it and u is 16-byte aligned
    bool ustage = pl.ustage && (reinterpret_cast<uintptr_t>(u) & 15) == 0;
    if (ustage) {
        EncodeTiledFn encode = encode_fn();
        if (!encode) return cudaErrorNotSupported;
        cuuint64_t gdim[2] = {32, (cuuint64_t)pl.batch * kw};
        cuuint64_t gstride[1] = {128};
        cuuint32_t box[2] = {32, kUBoxRows};
        cuuint32_t estride[2] = {1, 1};
        if (encode(&umap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(u), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    if (pl.tma) {
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
        } else {
            cuuint64_t gdim[2] = {(cuuint64_t)kw, (cuuint64_t)out};
            cuuint64_t gstride[1] = {(cuuint64_t)kw * 4};
            cuuint32_t box[2] = {kStepWords, 16};
            cuuint32_t estride[2] = {1, 1};
            if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(packed), gdim, gstride, box,
                       estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
    }
    for (int pass = 0; pass < pl.npass; ++pass) {
        for (int chunk = 0; chunk < pl.nchunk; ++chunk) {
            GemvArgs p;
            p.packed = packed;
            p.s = s;
            p.o = o;
            p.u = u;
            p.status = status;
            p.out = out;
            p.K = pl.K;
            p.kw = kw;
            p.c0 = pass * pl.cols;
            p.ncols = std::min(pl.cols, pl.batch - p.c0);
            p.kx0 = chunk * pl.kwc;
            p.kwc = pl.kwc;
            p.ngroups = (out + 15) / 16;
            p.maxgroups = pl.maxgroups;
            p.pitch = pl.pitch;
            p.image_bytes = (unsigned)pl.image_bytes;
            p.accumulate = chunk > 0;
            cudaError_t e = launch_planned(wmap, umap, ustage, p, pl, st);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace

DecodePlan make_decode_plan(int out, int K, int batch) {
    DecodePlan pl;
    memset(&pl, 0, sizeof(pl));
    if (out < 1 || K < 32 || K % 32 != 0 || batch < 1 || batch > 16) return pl;
    pl.out = out;
    pl.K = K;
    pl.kw = K / 32;
    pl.batch = batch;
    pl.row_bytes = (size_t)pl.kw * 16;
    // Measured on B200 (13824 x 12288 and 28672 x 20480 layers, GEMV back to
    // back): one and two columns are faster on the mma.sync kernel, four and
    // more on the tensor-core kernel, which reads every weight once whatever
    // the batch. At three columns mma.sync runs two passes (22.7 and 62.5 us)
    // against a tensor-core launch of ~24 us plus ~0.28 us per MB of weights
    // (30.0 and 44.8 us): the tensor-core kernel from 40 MB of packed weights.
    // Each takes the shapes the other cannot (the tensor-core kernel needs K a
    // multiple of 256 and at least 128 rows; the mma.sync kernel a word count
    // its planes fit).
    const double mbytes = (double)out * K / 8 / 1e6;
    pl.tc = (batch >= 4 || (batch == 3 && mbytes >= 40.0)) && plan_tc(pl);
    if (!pl.tc && !plan_mma(pl) && !(pl.tc = plan_tc(pl))) return pl;
    size_t off = 0;
    if (pl.tc) {
        // column summaries, word info, digit planes, group counters, partial slots
        pl.off_hdr = off;
        off = align256(off + (size_t)batch * pl.tc_nqp * 4);
        pl.off_steps = off;
        off = align256(off + (size_t)batch * pl.tc_kwp);
        pl.off_planes = off;
        off = align256(off + (size_t)pl.tc_n * pl.row_bytes);
        pl.off_count = off;
        off = align256(off + (size_t)pl.tc_groups * 4);
        pl.off_slots = off;
        off = align256(off + tc_slot_bytes(pl));
    } else {
        // the mma.sync kernel quantizes u inside each CTA and needs no scratch;
        // the workspace contract stays the same (a nonzero size means supported)
        off = 256;
        pl.off_hdr = pl.off_steps = pl.off_planes = pl.off_count = pl.off_slots = off;
    }
    pl.bytes = off;
    return pl;
}

size_t gemv_workspace_size(int out, int K, int batch) { return make_decode_plan(out, K, batch).bytes; }

cudaError_t launch_gemv(const uint32_t* packed, const float* s, int out, int K, const float* u, int batch, float* o,
                        void* ws, unsigned* status, cudaStream_t st) {
    const DecodePlan pl = make_decode_plan(out, K, batch);
    if (pl.bytes == 0) return cudaErrorInvalidValue;
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaError_t e;
    if (pl.tc) {
        e = launch_quant_mx(u, pl, w, st);
        if (e == cudaSuccess) e = launch_gemv_tc(packed, s, pl, o, w, status, st);
    } else {
        e = launch_mma(packed, s, pl, u, o, status, st);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_lift_gemv(const void* a, bool a_bf16, int batch, int in, const float* tinv, int tblk,
                             const float* M, int d, int D, const uint32_t* packed, const float* s, int out, int K,
                             float* u, float* o, void* ws, unsigned* status, cudaStream_t st) {
    cudaError_t e = launch_lift(a, a_bf16, batch, in, tinv, tblk, M, d, D, u, false, K, status, st);
    if (e != cudaSuccess) return e;
    return launch_gemv(packed, s, out, K, u, batch, o, ws, status, st);  // the quantizer waits for the lift
}

}  // namespace lq
