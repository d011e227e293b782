// Decode 1-bit GEMV on the fifth-generation tensor cores (LiftQuant paper note,
// "Key designs" 4: the 1-bit x float matmul with W_q after the small matmul
// T* a, then diag(s)), with u in the block-scaled 4-bit form of lq_decode.h:
//
//   o[c][r] = s[r] * 2^G_c * sum_p sum_k sigma[r][k] (d_p[c][k] / 2) 2^(E_w - 1 - 3p - G_c)
//
// The contraction is tcgen05.mma kind::mxf4 (e2m1 operands, ue8m0 scales per
// 32 elements, fp32 accumulation in tensor memory):
//   * A = the signs as e2m1 +-1.0: a sign word becomes four 32-bit registers of
//     eight nibbles (register r, nibble i <- bit r + 4i; one shift and one LOP3
//     each), stored into tensor memory with tcgen05.st (one row per lane), so
//     one M128 x K64 MMA consumes 8 KB of sign bits.
//   * B = the digit planes (row p * bpad + c: plane-major), TMA-loaded with the
//     128-byte swizzle, in the element order of the sign expansion.
//   * The scale of A is 1.0; the scale of B for row (p, c) and word w is
//     2^(E_w - 1 - 3p - G_c): written per sub-stage into tensor memory by the
//     warps that expand A (lane n % 32 of every quarter, column n / 32 of the
//     MMA's four-column group), from the words' exponents and the column maxima
//     G_c each CTA reduces from the quantizer's per-CTA summaries. Columns that
//     hold +-Inf use scale 1.0 for plane 0 of their Inf words and 2^-127 for
//     every other scale, so the accumulator holds (up to a negligible rest) the
//     count of +Inf terms minus -Inf terms of each row; NaN columns output NaN.
//   * Each M-tile has its own issuing warp. Measured on B200: a
//     tcgen05.commit releases its mbarrier only ~400 clocks after the MMAs it
//     covers, and one issuing thread's commits do not overlap, so a single
//     issuer committing every four small MMAs runs the tensor pipe at a third of
//     its rate; four issuers, each committing for its own tile, keep it busy.
//
// Work split: rows form groups of MT M-tiles of 128 (MT = 4 for narrow batches,
// 2 for wide ones, whose accumulators take more tensor memory), K sub-stages
// of 8 words (256 elements, four K64 MMAs per tile). The (group, sub-stage)
// units in group-major order are cut into one contiguous range per CTA, so every
// SM gets the same number of MMAs whatever the shape. The sign words arrive by
// TMA in stages of 32 words (128 bytes of each row, 128-byte swizzle), so DRAM
// serves whole 128-byte runs of a row; each stage feeds up to four sub-stages.
// A CTA's run inside one group is a segment; its accumulators are drained by
// the epilogue warps, which either store the result (the segment covers the
// whole group) or write a float64 partial to a workspace slot and count it in;
// the CTA that completes a group sums the partials in slot order
// (deterministic) and stores.
//   warp 0            TMA producer (weights, B, word info)
//   warps 1..4        sign expansion into TMEM A slots, B scale factors
//   warps 5..4+MT     one MMA issuer per M-tile (warp 5 also allocates TMEM)
//   last four warps   column info, accumulator drain, partials, results
// Every wait is bounded.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "lq_decode.h"
#include "lq_internal.h"
#include "lq_sm100.cuh"

namespace lq {
namespace {

using namespace sm100;

constexpr int kSub = 8;                             // words of K per sub-stage (4 MMAs of K64 per tile)
constexpr int kStageW = 32;                         // words of K per shared-memory stage (128 B per row)
constexpr int kMaxSS = 4;                           // shared-memory stages (at most)
constexpr int kMaxSA = 4;                           // tensor-memory A / scale slots (at most)
constexpr int kWTile = 128 * kStageW * 4;           // sign words of one M-tile in a stage: 16 KB
constexpr int kSFCols = 16;                         // TMEM columns of a slot's B scales (4 per MMA)
constexpr uint32_t kSpin = 1000000000u;             // bounded waits: 1 s

constexpr int kExpWarps = 8;                        // sign expansion: two warps per TMEM lane quarter

// warp 0 TMA, warps 1..8 expansion, MT issuers, four epilogue warps
__host__ __device__ constexpr int tc_threads(int MT) { return 32 * (1 + kExpWarps + MT + 4); }

struct TcArgs {
    const float* s;
    float* o;              // [batch][out]
    const uint32_t* summ;  // [batch][nqp] quantizer summaries
    unsigned* count;       // [groups] arrivals per group (cleared by the quantizer)
    double* slots;         // [groups][maxcontrib][batch][rows per group]
    unsigned* status;
    long long units;       // (group, sub-stage) units
    int out, kw, batch, bpad, N, nq, nqp, groups, nsub, maxcontrib, nacc, nss, nsa;
};

struct Smem {
    size_t b, w, info, col, flag, bars, total;
    size_t bstage, istage, isumm;
};

// Per stage: B (four sub-stage tiles of N rows x 128 B), the sign words of MT
// tiles, and per column the 32 word deltas and the 4 quantizer summaries of
// the stage (each region 128-byte aligned).
__host__ __device__ inline Smem tc_smem(int MT, int N, int batch, int nss) {
    Smem L;
    L.bstage = (size_t)4 * N * 128;
    L.isumm = ((size_t)batch * kStageW + 127) & ~(size_t)127;
    L.istage = L.isumm + (((size_t)batch * 16 + 127) & ~(size_t)127);
    L.b = 0;
    L.w = L.b + nss * L.bstage;                        // multiples of 1024 (N is a multiple of 8)
    L.info = L.w + (size_t)nss * MT * kWTile;
    L.col = L.info + nss * L.istage;
    L.flag = L.col + 16 * 16;  // per column: G (biased), mode, Inf count
    L.bars = L.flag + 16;
    L.total = L.bars + 8 * (3 * kMaxSS + 2 * kMaxSA + 4 + 4) + 1024 /*alignment slack*/;
    return L;
}

// Tensor-memory columns of the accumulators, A slots, B scale slots and A scales.
__host__ __device__ inline int tc_tmem_cols(int MT, int N, int nacc, int nsa) {
    return ((nacc * MT * N + 31) & ~31) + nsa * (MT * 32 + kSFCols) + 16;
}

// floor(i * n / parts) in 64-bit
__device__ __forceinline__ long long split_at(long long i, long long n, long long parts) { return i * n / parts; }

// The CTA whose range holds unit x.
__device__ __forceinline__ int cta_of(long long x, long long units, int grid) {
    int b = (int)(x * grid / units);
    while (b > 0 && split_at(b, units, grid) > x) --b;
    while (b + 1 < grid && split_at(b + 1, units, grid) <= x) ++b;
    return b;
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// Sum the kMxPlanes plane columns (p * BP + c) of one accumulator tile into
// part[c], c < BP: the tile's columns read 32 at a time.
template <int BP, int C>
__device__ __forceinline__ void drain_tile(uint32_t taddr, double (&part)[C]) {
    static_assert(BP <= C, "plane columns beyond the partial sums");
    constexpr int kCols = kMxPlanes * BP;
    if constexpr (BP <= 4) {  // up to 28 columns: one load
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < kCols; ++e) part[e % BP] += (double)__uint_as_float(v[e]);
    } else {  // 16 columns at a time (fewer live registers beside the 16 partial sums)
#pragma unroll
        for (int ch = 0; ch < (kCols + 15) / 16; ++ch) {
            uint32_t v[16];
            tmem_ld_x16(taddr + 16 * ch, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e)
                if (16 * ch + e < kCols) part[(16 * ch + e) % BP] += (double)__uint_as_float(v[e]);
        }
    }
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::mxf4 with ue8m0 block scales of 32.
__device__ __forceinline__ void umma_mxf4(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                          uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], [%1], %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// e2m1 +-1.0 nibbles of a sign word: register r, nibble i <- bit r + 4i.
__device__ __forceinline__ void expand_word(uint32_t w, uint32_t* v) {
    v[0] = (~(w << 3) & 0x88888888u) | 0x22222222u;
    v[1] = (~(w << 2) & 0x88888888u) | 0x22222222u;
    v[2] = (~(w << 1) & 0x88888888u) | 0x22222222u;
    v[3] = (~w & 0x88888888u) | 0x22222222u;
}

__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// Instruction descriptor, kind::mxf4: A, B e2m1, ue8m0 scales, K-major, M = 128.
__device__ __forceinline__ uint32_t idesc_mxf4(int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | (8u << 24);
}

// Walks a CTA's sub-stages: unit -> (group, sub-stage), the index ks of its
// shared-memory stage in the CTA's sequence (a new stage starts at every
// 32-word boundary and at every group) with its ring slot ks % nss and phase
// (ks / nss) & 1 kept incrementally, and whether it is the last sub-stage of
// that stage or of its group segment.
struct Walker {
    long long u0, u1;
    int nsub, nss;
    long long g;
    int sub, ks, slot, phase;
    __device__ void init(long long a, long long b, int n, int stages) {
        u0 = a;
        u1 = b;
        nsub = n;
        nss = stages;
        g = a / n;
        sub = (int)(a - g * n);
        ks = slot = phase = 0;
    }
    __device__ bool seg_first(long long u) const { return u == u0 || sub == 0; }
    __device__ bool seg_last(long long u) const { return u + 1 == u1 || sub + 1 == nsub; }
    __device__ bool stage_last(long long u) const { return seg_last(u) || ((sub + 1) & 3) == 0; }
    __device__ void next(long long u) {
        const bool new_stage = stage_last(u);
        if (sub + 1 == nsub) {
            ++g;
            sub = 0;
        } else {
            ++sub;
        }
        if (new_stage) {
            ++ks;
            if (++slot == nss) {
                slot = 0;
                phase ^= 1;
            }
        }
    }
};

// Index and phase of a ring of n slots, advanced one use at a time.
struct Ring {
    int idx, phase, n;
    __device__ void init(int slots) {
        idx = phase = 0;
        n = slots;
    }
    __device__ void next() {
        if (++idx == n) {
            idx = 0;
            phase ^= 1;
        }
    }
};

template <int MT>
__global__ void __launch_bounds__(tc_threads(MT), 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap bmap,
                   const __grid_constant__ CUtensorMap dmap, const __grid_constant__ CUtensorMap smap,
                   const TcArgs p) {
    constexpr int kRG = 128 * MT;       // rows per group
    constexpr int kACols = MT * 32;     // TMEM columns of an A slot
    constexpr int kIss0 = 1 + kExpWarps;  // first issuer warp (it also owns the TMEM allocation)
    constexpr int kEpi0 = kIss0 + MT;     // first epilogue warp
    constexpr int kNamed1 = 32 * (kExpWarps + 4);  // expansion + epilogue warps
    constexpr int kCmax = MT == 4 ? 4 : 16;        // batch columns (four M-tiles serve at most four)
    // the next kernel on the stream (the next layer's lift or quantizer) waits for
    // this grid before it reads anything; it may be scheduled as SMs free up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const Smem L = tc_smem(MT, p.N, p.batch, p.nss);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nss = p.nss, nsa = p.nsa;
    int* col = reinterpret_cast<int*>(smem + L.col);        // [c][4]: biased G, mode, Inf count
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flag);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.flag + 4);
    const uint32_t bars = smem_addr(smem + L.bars);
    const uint32_t full_w = bars, full_b = bars + 8 * kMaxSS, freed = bars + 16 * kMaxSS;
    const uint32_t a_full = bars + 24 * kMaxSS, a_empty = a_full + 8 * kMaxSA;
    const uint32_t acc_full = a_empty + 8 * kMaxSA, acc_empty = acc_full + 16, done = acc_empty + 16;

    const long long u0 = split_at(blockIdx.x, p.units, gridDim.x), u1 = split_at(blockIdx.x + 1, p.units, gridDim.x);

    if (threadIdx.x == 0) {
        for (int st = 0; st < nss; ++st) {
            mbar_init(full_w + 8 * st, 1);
            mbar_init(full_b + 8 * st, 1);
            mbar_init(freed + 8 * st, kExpWarps + MT);  // the expansion warps read it, MT issuers consumed it
        }
        for (int a = 0; a < nsa; ++a) {
            mbar_init(a_full + 8 * a, kExpWarps);  // the expansion warps wrote every tile and the scales
            mbar_init(a_empty + 8 * a, MT);      // every issuer's MMAs on it completed
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full + 8 * b, MT);
            mbar_init(acc_empty + 8 * b, 4);
        }
        for (int t = 0; t < MT; ++t) mbar_init(done + 8 * t, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&wmap);
        prefetch_tensormap(&bmap);
        prefetch_tensormap(&dmap);
        prefetch_tensormap(&smap);
    }
    if (warp == kIss0) {
        tmem_alloc(smem_addr(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t acol0 = (uint32_t)(p.nacc * MT * p.N + 31) & ~31u;
    const uint32_t sfcol0 = acol0 + nsa * kACols, sfacol = sfcol0 + nsa * kSFCols;

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            Walker wk;
            wk.init(u0, u1, p.nsub, nss);
            auto issue_w = [&](int slot, long long g, int stg) {
                mbar_arrive_expect_tx(full_w + 8 * slot, MT * kWTile);
                for (int t = 0; t < MT; ++t)
                    tma_load_2d(smem_addr(smem + L.w + ((size_t)slot * MT + t) * kWTile), &wmap, stg * kStageW,
                                (int)(g * kRG) + 128 * t, full_w + 8 * slot);
            };
            auto issue_b = [&](int slot, int stg) {
                const uint32_t ib = smem_addr(smem + L.info + slot * L.istage);
                mbar_arrive_expect_tx(full_b + 8 * slot, (uint32_t)(L.bstage + p.batch * (kStageW + 16)));
                tma_load_3d(smem_addr(smem + L.b + slot * L.bstage), &bmap, 0, 0, stg * 4, full_b + 8 * slot);
                tma_load_2d(ib, &dmap, stg * kStageW, 0, full_b + 8 * slot);
                tma_load_2d(ib + (uint32_t)L.isumm, &smap, stg * 4, 0, full_b + 8 * slot);
            };
            // the sign words do not depend on the kernel before this one: request
            // the first stages before waiting for it
            int early = 0;
            {
                Walker e = wk;
                for (long long u = u0; u < u1 && early < nss; ++u) {
                    if (e.stage_last(u)) {
                        issue_w(early, e.g, e.sub >> 2);
                        ++early;
                    }
                    e.next(u);
                }
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");
            int issued = 0;  // stages whose B was requested
            for (long long u = u0; u < u1; ++u) {
                if (wk.stage_last(u)) {
                    const int ks = wk.ks, slot = wk.slot;
                    if (ks >= nss) {
                        if (!mbar_wait(freed + 8 * slot, wk.phase ^ 1, p.status, kSpin)) {
                            *abort_flag = 1;
                            break;
                        }
                        issue_w(slot, wk.g, wk.sub >> 2);
                    }
                    issue_b(slot, wk.sub >> 2);
                    issued = ks + 1;
                }
                wk.next(u);
            }
            // leave no copy in flight: wait (bounded) for the last loads of each slot
            const int total = max(issued, early);
            for (int ks = max(0, total - nss); ks < total; ++ks) {
                mbar_wait(full_w + 8 * (ks % nss), (ks / nss) & 1, p.status, kSpin);
                if (ks < issued) mbar_wait(full_b + 8 * (ks % nss), (ks / nss) & 1, p.status, kSpin);
            }
        }
    } else if (warp <= kExpWarps) {
        // ================================================================ sign expansion, B scales
        // Each lane quarter's 32 rows of the MT tiles are split between its two
        // warps k: warp k expands tiles k MT/2 .. (k+1) MT/2 - 1 and writes the B
        // scales of MMAs kk = 2k, 2k + 1 (words 4k .. 4k + 3 of the sub-stage).
        // More warps do not help: the tensor-memory stores of the expanded
        // operand (four bytes per sign byte) set the pace.
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int k = (warp - 1) >> 2;          // 0..1
        const int r = 32 * q + lane;            // row within each M-tile
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        if (k == 0) {  // A scales: 1.0 for every row and block
            uint32_t one[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) one[x] = 0x7F7F7F7Fu;
            tmem_st_x16(lane_base + sfacol, one);
        }
        named_bar(1, kNamed1);  // column info from the epilogue warps
        // this lane's B rows n = 32 c4 + lane: column, scale base 126 - 3p - G_c (biased), mode
        // (four M-tiles serve at most four columns: 28 B rows, one block of 32)
        constexpr int kRB = MT == 4 ? 1 : 4;
        int rc[kRB], rbase[kRB], rmode[kRB];
        bool rp0[kRB];
#pragma unroll
        for (int c4 = 0; c4 < kRB; ++c4) {
            const int n = 32 * c4 + lane;
            const int pl = n / p.bpad, c = n - pl * p.bpad;
            const bool live = n < p.N && pl < kMxPlanes && c < p.batch;
            rc[c4] = live ? c : 0;
            rmode[c4] = live ? col[4 * c + 1] : -1;
            rbase[c4] = live ? 126 - 3 * pl - col[4 * c] : 0;
            rp0[c4] = pl == 0;
        }
        const int nrows4 = (p.N + 31) / 32;  // row blocks of 32 that hold B rows
        Walker wk;
        wk.init(u0, u1, p.nsub, nss);
        Ring ar;
        ar.init(nsa);
        int i = 0;
        for (long long u = u0; u < u1; ++u, ++i, ar.next()) {
            const int slot = wk.slot, j = wk.sub & 3, a = ar.idx;
            bool ok = mbar_wait(full_w + 8 * slot, wk.phase, p.status, kSpin);
            ok = ok && mbar_wait(full_b + 8 * slot, wk.phase, p.status, kSpin);
            ok = ok && (i < nsa || mbar_wait(a_empty + 8 * a, ar.phase ^ 1, p.status, kSpin));
            if (!__all_sync(0xffffffffu, ok) || *abort_flag) {  // tcgen05.st is warp-collective
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            // ---- A: the 8 words of row r of this warp's tiles (128-byte swizzle:
            // 16-byte chunk c at c ^ (r & 7))
#pragma unroll
            for (int tt = 0; tt < MT / 2; ++tt) {
                const int t = k * (MT / 2) + tt;
                const uint8_t* row = smem + L.w + ((size_t)slot * MT + t) * kWTile + (size_t)r * 128;
                const uint4 w0 = *reinterpret_cast<const uint4*>(row + (((2 * j) ^ (r & 7)) << 4));
                const uint4 w1 = *reinterpret_cast<const uint4*>(row + (((2 * j + 1) ^ (r & 7)) << 4));
                uint32_t v[32];
                expand_word(w0.x, v);
                expand_word(w0.y, v + 4);
                expand_word(w0.z, v + 8);
                expand_word(w0.w, v + 12);
                expand_word(w1.x, v + 16);
                expand_word(w1.y, v + 20);
                expand_word(w1.z, v + 24);
                expand_word(w1.w, v + 28);
                tmem_st_32x32b_x32(lane_base + acol0 + a * kACols + t * 32, v);
            }
            // ---- B scales of MMAs kk = 2k, 2k + 1: words 8 j + 4k .. + 3 of each live
            // row's column; scale column 4 kk + c4, bytes 0 and 1 for the MMA's two
            // blocks of 32
            const uint8_t* dsm = smem + L.info + slot * L.istage;
            const uint32_t* ssm = reinterpret_cast<const uint32_t*>(dsm + L.isumm);
            uint32_t sf[8] = {0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu,
                              0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu};
            // every row block's loads first (rows without a B row read column 0)
            uint32_t dlv[kRB], elv[kRB];
#pragma unroll
            for (int c4 = 0; c4 < kRB; ++c4) {
                dlv[c4] = *reinterpret_cast<const uint32_t*>(dsm + rc[c4] * kStageW + 8 * j + 4 * k);
                elv[c4] = ssm[4 * rc[c4] + j] & kInfoExp;
            }
#pragma unroll
            for (int c4 = 0; c4 < kRB; ++c4) {
                uint32_t e4 = 0x7F7F7F7Fu;  // rows without a B row: any finite scale
                if (c4 < nrows4 && rmode[c4] >= 0) {
                    const uint32_t dl = dlv[c4];
                    if (rmode[c4] == kColFinite) {
                        // 2^(E - 1 - 3p - G_c): base 126 - 3p - (G_c - E_loc), less each word's delta
                        const int base = max(0, rbase[c4] + (int)elv[c4]);
                        // per byte max(0, base - delta), both below 128: (base | 0x80) - delta
                        // stays within each byte, its bit 7 tells the sign
                        const uint32_t t4 = ((uint32_t)base * 0x01010101u | 0x80808080u) - (dl & 0x7F7F7F7Fu);
                        const uint32_t pos = (t4 >> 7) & 0x01010101u;
                        e4 = t4 & 0x7F7F7F7Fu & (pos * 0xFFu);
                    } else if (rmode[c4] == kColInf) {
                        e4 = rp0[c4] ? ((dl >> 7) & 0x01010101u) * 127u : 0u;  // plane 0 of Inf words: 1.0
                    }
                }
                sf[c4] = __byte_perm(e4, 0x7F7F7F7Fu, 0x4410);      // words 0, 1 of the four: MMA kk = 2k
                sf[4 + c4] = __byte_perm(e4, 0x7F7F7F7Fu, 0x4432);  // words 2, 3: MMA kk = 2k + 1
            }
            tmem_st_x8(lane_base + sfcol0 + a * kSFCols + 8 * k, sf);
            __syncwarp();
            if (lane == 0 && wk.stage_last(u)) mbar_arrive(freed + 8 * slot);  // read all it needs from the stage
            tmem_st_wait();
            tc_fence_before();
            if (lane == 0) mbar_arrive(a_full + 8 * a);
            wk.next(u);
        }
    } else if (warp < kEpi0) {
        // ================================================================ MMA issuer of M-tile t
        const int t = warp - kIss0;
        if (lane == 0) {
            const uint32_t idesc = idesc_mxf4(p.N);
            int buf = 0;
            int uses[2] = {0, 0};
            Walker wk;
            wk.init(u0, u1, p.nsub, nss);
            Ring ar;
            ar.init(nsa);
            for (long long u = u0; u < u1; ++u, ar.next()) {
                const bool first = wk.seg_first(u), last = wk.seg_last(u);
                const int slot = wk.slot, j = wk.sub & 3, a = ar.idx;
                bool ok = true;
                if (first && uses[buf] > 0) ok = mbar_wait(acc_empty + 8 * buf, (uses[buf] - 1) & 1, p.status, kSpin);
                ok = ok && mbar_wait(full_b + 8 * slot, wk.phase, p.status, kSpin);
                ok = ok && mbar_wait(a_full + 8 * a, ar.phase, p.status, kSpin);
                if (!ok || *abort_flag) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint64_t bdesc = smem_desc_sw128(smem_addr(smem + L.b + slot * L.bstage + (size_t)j * p.N * 128));
                const uint32_t acc = tmem + (uint32_t)((buf * MT + t) * p.N);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_mxf4(acc, tmem + acol0 + a * kACols + t * 32 + kk * 8, bdesc + (uint64_t)((kk * 32) >> 4),
                              idesc, tmem + sfacol, tmem + sfcol0 + a * kSFCols + 4 * kk, (uint32_t)(!first || kk > 0));
                umma_commit(a_empty + 8 * a);
                if (wk.stage_last(u)) umma_commit(freed + 8 * slot);
                if (last) {
                    umma_commit(acc_full + 8 * buf);
                    ++uses[buf];
                    buf = p.nacc == 2 ? buf ^ 1 : 0;
                }
                wk.next(u);
            }
            umma_commit(done + 8 * t);  // fires when every MMA issued above has completed
            mbar_wait(done + 8 * t, 0, p.status, kSpin);
        }
    } else {
        // ================================================================ column info, drain, results
        const int q = warp & 3;
        const int et = threadIdx.x - 32 * kEpi0;  // 0..127
        asm volatile("griddepcontrol.wait;" ::: "memory");
        // column info: biased max exponent, mode, Inf count, from the per-CTA summaries
        for (int c = warp - kEpi0; c < p.batch; c += 4) {
            uint32_t e = 0, f = 0, n = 0;
            for (int jj = lane; jj < p.nq; jj += 32) {
                const uint32_t v = p.summ[(size_t)c * p.nqp + jj];
                e = max(e, v & kInfoExp);
                f |= v & (kInfoNaN | kInfoInf);
                n += v >> 16;
            }
            e = __reduce_max_sync(0xffffffffu, e);
            f = __reduce_or_sync(0xffffffffu, f);
            n = __reduce_add_sync(0xffffffffu, n);
            if (lane == 0) {
                col[4 * c] = (int)e;
                col[4 * c + 1] = (f & kInfoNaN) ? kColNaN : (f & kInfoInf) ? kColInf : kColFinite;
                col[4 * c + 2] = (int)n;
            }
        }
        named_bar(1, kNamed1);
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L.flag + 8);
        int buf = 0, use[2] = {0, 0};
        long long u = u0;
        while (u < u1) {
            const long long g = u / p.nsub;
            const long long uend = min(u1, (g + 1) * p.nsub);
            // contributors of group g: the CTAs holding its first and last unit
            const int bfirst = cta_of(g * p.nsub, p.units, gridDim.x);
            const int blast = cta_of((g + 1) * p.nsub - 1, p.units, gridDim.x);
            const int nc = blast - bfirst + 1, jslot = (int)blockIdx.x - bfirst;
            const bool ok = mbar_wait(acc_full + 8 * buf, use[buf] & 1, p.status, kSpin);
            if (!__all_sync(0xffffffffu, ok)) *abort_flag = 1;
            // the four warps decide together (they meet at named barriers below)
            named_bar(2, 128);
            if (et == 0) *last_flag = *abort_flag;
            named_bar(2, 128);
            if (*last_flag) break;
            tc_fence_after();
            double* slot = p.slots + ((size_t)(g * p.maxcontrib + jslot) * p.batch) * kRG;
            // store the results of tile t of group g from the plane sums x[c]
            auto store_tile = [&](int t, const double (&x)[kCmax]) {
                const long long r = g * kRG + t * 128 + 32 * q + lane;
                if (r >= p.out) return;
                const double sr = (double)__ldg(p.s + r);
#pragma unroll
                for (int c = 0; c < kCmax; ++c) {
                    if (c >= p.batch) continue;
                    const int mode = col[4 * c + 1];
                    float res;
                    if (mode == kColFinite) {
                        // undo the column normalization 2^-G_c (G_c = biased - kMxBias)
                        const double scale = __longlong_as_double((long long)(col[4 * c] - kMxBias + 1023) << 52);
                        res = (float)(x[c] * scale * sr);
                    } else if (mode == kColInf) {
                        const double S = rint(x[c]);
                        const double n = (double)col[4 * c + 2];
                        const double inf = __longlong_as_double(0x7ff0000000000000ll);
                        const double val = S == n ? inf : S == -n ? -inf : __longlong_as_double(0x7ff8000000000000ll);
                        res = (float)(val * sr);
                    } else {
                        res = __int_as_float(0x7fc00000);
                    }
                    p.o[(size_t)c * p.out + r] = res;
                }
            };
            // ---- drain tile by tile: sum the planes of each column (plane p =
            // columns p * bpad ..), then store the result (the group is this
            // CTA's alone) or the partial to slot (g, jslot)
#pragma unroll 1
            for (int t = 0; t < MT; ++t) {
                double part[kCmax];
#pragma unroll
                for (int c = 0; c < kCmax; ++c) part[c] = 0.0;
                const uint32_t tacc = lane_base + (uint32_t)((buf * MT + t) * p.N);
                if (p.bpad == 1) {
                    drain_tile<1>(tacc, part);
                } else if (p.bpad == 2) {
                    drain_tile<2>(tacc, part);
                } else if (p.bpad == 4 || MT == 4) {
                    drain_tile<4>(tacc, part);
                } else if constexpr (MT == 2) {
                    if (p.bpad == 8)
                        drain_tile<8>(tacc, part);
                    else
                        drain_tile<16>(tacc, part);
                }
                if (nc == 1) {
                    store_tile(t, part);
                } else {
#pragma unroll
                    for (int c = 0; c < kCmax; ++c)
                        if (c < p.batch) slot[(size_t)c * kRG + t * 128 + 32 * q + lane] = part[c];
                }
            }
            tc_fence_before();
            if (lane == 0) mbar_arrive(acc_empty + 8 * buf);
            ++use[buf];
            buf = p.nacc == 2 ? buf ^ 1 : 0;

            if (nc > 1) {
                // the CTA that completes group g sums the partials in slot order
                __threadfence();
                named_bar(2, 128);
                if (et == 0) {
                    const unsigned old = atomicAdd(p.count + g, 1u);
                    const int last = old == (unsigned)(nc - 1);
                    if (last) p.count[g] = 0u;
                    *last_flag = last;
                }
                named_bar(2, 128);
                if (*last_flag != 0) {
                    __threadfence();
                    const double* base = p.slots + ((size_t)(g * p.maxcontrib) * p.batch) * kRG;
#pragma unroll 1
                    for (int t = 0; t < MT; ++t) {
                        // slot order outside, columns inside: each round issues the
                        // loads of every column at once
                        double sum[kCmax];
#pragma unroll
                        for (int c = 0; c < kCmax; ++c) sum[c] = 0.0;
#pragma unroll 1
                        for (int jj = 0; jj < nc; ++jj) {
                            const double* sj = base + (size_t)jj * p.batch * kRG + t * 128 + 32 * q + lane;
                            double x[kCmax];
#pragma unroll
                            for (int c = 0; c < kCmax; ++c) x[c] = c < p.batch ? __ldcg(sj + (size_t)c * kRG) : 0.0;
#pragma unroll
                            for (int c = 0; c < kCmax; ++c) sum[c] += x[c];
                        }
                        store_tile(t, sum);
                    }
                }
            }
            u = uend;
        }
    }

    // lane 0 of several warps ran its role alone: reconverge every warp before
    // the CTA barrier that orders the TMEM release after all tensor-memory use
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == kIss0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_tc() {
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

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

}  // namespace

bool plan_tc(DecodePlan& p) {
    // whole 128-byte chunks of digit rows per sub-stage (K a multiple of 256) and
    // boxes no taller than the tensor (at least one M-tile of rows)
    if (p.kw % kSub != 0 || p.batch > 16 || p.out < 128) return false;
    int bpad = 1;
    while (bpad < p.batch) bpad *= 2;
    p.tc_bpad = bpad;
    p.tc_n = (kMxPlanes * bpad + 7) / 8 * 8;
    // tiles per group (four issuers when the accumulators allow), A / scale slots
    // (at least two), accumulator buffers: the first that fits tensor memory
    p.tc_mt = 0;
    for (int mt = bpad <= 4 ? 4 : 2; mt >= 2 && !p.tc_mt; mt -= 2)
        for (int nsa = kMaxSA; nsa >= 2 && !p.tc_mt; --nsa)
            for (int nacc = 2; nacc >= 1; --nacc)
                if (tc_tmem_cols(mt, p.tc_n, nacc, nsa) <= 512) {
                    p.tc_mt = mt;
                    p.tc_nsa = nsa;
                    p.tc_nacc = nacc;
                    break;
                }
    if (!p.tc_mt) return false;
    const int rg = 128 * p.tc_mt;
    p.tc_groups = (p.out + rg - 1) / rg;
    p.tc_stages = (p.kw + kSub - 1) / kSub;  // sub-stages per group
    p.tc_units = (long long)p.tc_groups * p.tc_stages;
    p.tc_grid = (int)std::min<long long>(sm_count(), p.tc_units);
    p.tc_nq = (p.kw + kMxQWords - 1) / kMxQWords;
    p.tc_nqp = (p.tc_nq + 3) & ~3;   // 16-byte rows for the summary copies
    p.tc_kwp = (p.kw + 15) & ~15;    // 16-byte rows for the delta copies
    // shared memory: as many stages as fit, up to kMaxSS
    p.tc_nss = 0;
    for (int nss = kMaxSS; nss >= 2; --nss)
        if (tc_smem(p.tc_mt, p.tc_n, p.batch, nss).total <= 227 * 1024) {
            p.tc_nss = nss;
            break;
        }
    if (!p.tc_nss) return false;
    p.tc_smem = tc_smem(p.tc_mt, p.tc_n, p.batch, p.tc_nss).total;
    // most CTAs that share one group
    auto cta_of_h = [&](long long x) {
        long long b = x * p.tc_grid / p.tc_units;
        while (b > 0 && b * p.tc_units / p.tc_grid > x) --b;
        while (b + 1 < p.tc_grid && (b + 1) * p.tc_units / p.tc_grid <= x) ++b;
        return b;
    };
    int maxc = 1;
    for (long long g = 0; g < p.tc_groups; ++g) {
        const long long nc = cta_of_h((g + 1) * p.tc_stages - 1) - cta_of_h(g * p.tc_stages) + 1;
        maxc = std::max<int>(maxc, (int)nc);
    }
    p.tc_maxcontrib = maxc;
    return true;
}

size_t tc_slot_bytes(const DecodePlan& p) {
    return p.tc_maxcontrib > 1 ? (size_t)p.tc_groups * p.tc_maxcontrib * p.batch * (128 * p.tc_mt) * sizeof(double) : 0;
}

cudaError_t launch_gemv_tc(const uint32_t* packed, const float* s, const DecodePlan& pl, float* o, uint8_t* ws,
                           unsigned* status, cudaStream_t st) {
    EncodeTiledFn encode = encode_fn_tc();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap wmap, bmap, dmap, smap;
    {  // sign words [out][kw], box 32 words (128 B) x 128 rows, 128-byte swizzle
        cuuint64_t gdim[2] = {(cuuint64_t)pl.kw, (cuuint64_t)pl.out};
        cuuint64_t gstride[1] = {(cuuint64_t)pl.kw * 4};
        cuuint32_t box[2] = {kStageW, 128};
        cuuint32_t es[2] = {1, 1};
        if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(packed), gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {  // digit planes [N rows][K / 2 bytes] as [chunk of 128 B][row][byte]: box 128 B x N rows x 4 chunks
       // (the four sub-stages of a stage), 128-byte swizzle; rows past kMxPlanes * bpad are unused
        cuuint64_t gdim[3] = {128, (cuuint64_t)pl.tc_n, (cuuint64_t)pl.tc_stages};
        cuuint64_t gstride[2] = {(cuuint64_t)pl.row_bytes, 128};
        cuuint32_t box[3] = {128, (cuuint32_t)pl.tc_n, 4};
        cuuint32_t es[3] = {1, 1, 1};
        if (encode(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, ws + pl.off_planes, gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {  // word deltas [batch][kwp] bytes, box 32 words x batch
        cuuint64_t gdim[2] = {(cuuint64_t)pl.tc_kwp, (cuuint64_t)pl.batch};
        cuuint64_t gstride[1] = {(cuuint64_t)pl.tc_kwp};
        cuuint32_t box[2] = {kStageW, (cuuint32_t)pl.batch};
        cuuint32_t es[2] = {1, 1};
        if (encode(&dmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, ws + pl.off_steps, gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {  // quantizer summaries [batch][nqp], box 4 (the sub-stages of a stage) x batch
        cuuint64_t gdim[2] = {(cuuint64_t)pl.tc_nqp, (cuuint64_t)pl.batch};
        cuuint64_t gstride[1] = {(cuuint64_t)pl.tc_nqp * 4};
        cuuint32_t box[2] = {4, (cuuint32_t)pl.batch};
        cuuint32_t es[2] = {1, 1};
        if (encode(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, ws + pl.off_hdr, gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    TcArgs a;
    a.s = s;
    a.o = o;
    a.summ = reinterpret_cast<const uint32_t*>(ws + pl.off_hdr);
    a.count = reinterpret_cast<unsigned*>(ws + pl.off_count);
    a.slots = reinterpret_cast<double*>(ws + pl.off_slots);
    a.status = status;
    a.units = pl.tc_units;
    a.out = pl.out;
    a.kw = pl.kw;
    a.batch = pl.batch;
    a.bpad = pl.tc_bpad;
    a.N = pl.tc_n;
    a.nq = pl.tc_nq;
    a.nqp = pl.tc_nqp;
    a.groups = pl.tc_groups;
    a.nsub = pl.tc_stages;
    a.maxcontrib = pl.tc_maxcontrib;
    a.nacc = pl.tc_nacc;
    a.nss = pl.tc_nss;
    a.nsa = pl.tc_nsa;

    auto kern = pl.tc_mt == 4 ? gemv_tc_kernel<4> : gemv_tc_kernel<2>;
    static size_t granted[2][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int ki = pl.tc_mt == 4 ? 1 : 0;
    if (dev >= 64 || granted[ki][dev] < pl.tc_smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.tc_smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) granted[ki][dev] = pl.tc_smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.tc_grid, 1, 1);
    cfg.blockDim = dim3(tc_threads(pl.tc_mt), 1, 1);
    cfg.dynamicSmemBytes = pl.tc_smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, wmap, bmap, dmap, smap, a);
}

}  // namespace lq
