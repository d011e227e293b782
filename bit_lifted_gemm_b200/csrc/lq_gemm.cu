// Prefill 1-bit GEMM on the fifth-generation tensor cores (LiftQuant paper
// note, "Key designs" 4: the layer is a 1-bit x float matmul with W_q after the
// small matmul T* a, then diag(s)):
//
//   o[t][r] = s[r] * sum_k sigma[r][k] u[t][k]
//
// Prefill is a dense contraction, so it runs on tcgen05 with bf16 operands and
// fp32 accumulation in tensor memory. +-1 is exact in bf16 and every product
// is exact; the only rounding is fp32 accumulation (plus the bf16 rounding of
// u done by the lift).
//
// One CTA computes a 128 (rows of W_q) x BN (tokens) tile, K in steps of 64;
// BN = 256, or 64 for short token runs (a quarter of the MMA, TMEM and u
// traffic per k-step). When the tiles cannot fill the SMs, K is split in two:
// each half scales its partial by s[r] and adds it atomically into o, zeroed
// first; with exactly two terms the sum does not depend on their order, so
// the result is deterministic.
//   warp 0      TMA producer: u tile [BN tokens][64 k] bf16, 128-byte swizzle
//   warp 1      TMEM allocator and single-thread UMMA issuer (M=128, N=BN, K=16)
//   warps 2..5  one thread per tile row: load that row's two sign words for the
//               k-step, expand the 64 bits to +-1 bf16 in registers and store
//               them in the same 128-byte-swizzled K-major layout the TMA uses;
//               after the K loop the same warps drain TMEM (tcgen05.ld), apply
//               s[r] and store o.
// A 4-stage mbarrier ring couples them; the unpackers fence the generic-proxy
// stores into the async proxy before arriving. Every wait is bounded.
#include <cuda.h>

#include "lq_debug.cuh"
#include "lq_internal.h"
#include "lq_sm100.cuh"

namespace lq {
namespace {

using namespace sm100;

constexpr int BM = 128, BK = 64, STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;   // 16 KB
constexpr int A_COLS = BK / 2;         // TMEM columns of one A stage (two bf16 per 32-bit column)
constexpr int THREADS = 192;
constexpr int UNPACK_THREADS = 128;
template <int BN>
struct Tile {
    static constexpr int B_STAGE = BN * BK * 2;  // 32 KB (BN 256) or 8 KB (BN 64)
    static constexpr int TMEM_COLS = BN;         // fp32 accumulator, 128 lanes x BN columns
    static constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * (A_STAGE + B_STAGE) + 256;
};
// The variant for short token runs keeps the A stages in TMEM after the
// accumulators (the unpackers store them with tcgen05.st; no A traffic through
// shared memory): measured faster for 64-token tiles, slower for 256-token ones.
// Its k-steps alternate between NI issuing threads in separate warps, each with
// an accumulator of its own: one thread's commits complete one after another,
// ~400 clocks apart, longer than the four MMAs of a 64-token k-step take.
template <int BN, int NI, int S>
struct TileTA {
    static constexpr int A_COL = BN * NI;
    static constexpr int TMEM_COLS = A_COL + S * A_COLS <= 256 ? 256 : 512;  // a power of two
    static constexpr int THREADS = 32 * (6 + NI - 1);  // issuers past the first are warps 6, 7, ...
    static constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + S * Tile<BN>::B_STAGE + 256;
    static_assert(A_COL + S * A_COLS <= 512, "accumulators and A stages exceed tensor memory");
};
constexpr int TA_ISSUERS = 2, TA_STAGES = 4;

// Expand 16 sign bits (bit i = element i of a k-run) into 8 bf16x2 words:
// word i holds elements (2i, 2i+1) as +1.0 (0x3F80) or -1.0 (0xBF80).
// Even bits stay, odd bits move up by 15 so that one shift brings bits 2i and
// 2i+1 to the two sign positions (15 and 31).
__device__ __forceinline__ void expand16(uint32_t x, uint32_t* v) {
    const uint32_t q = (x & 0x5555u) | ((x & 0xAAAAu) << 15);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = ((q << (15 - 2 * i)) & 0x80008000u) ^ 0xBF80BF80u;
}

// Tiled 2-D bulk store of a shared-memory box into global memory, and the same
// with an element-wise add into global memory (f32); both complete in a bulk
// group of the issuing thread.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map), "r"(src),
                 "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     map),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every bulk store of this thread is complete.
__device__ __forceinline__ void bulk_wait_group_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Named barrier over `nthreads` threads (whole warps).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// Epilogue of both kernels, run by the four warps that own the TMEM lane
// quarters (warp & 3): o[t][r] = s[r] * (sum of the nacc accumulators, columns
// acc_stride apart, added in order) for the 128 x BN tile at (m0, n0). With a
// tensor map for o the warps stage the tile in shared memory ([BN][128] fp32,
// in the operand stages, idle once the accumulators are final) and one thread
// writes it with one TMA store, or with a TMA add when K is split (two addends
// into a zeroed o: the same sum in either order); rows and tokens past the
// tensor are clipped. Without one (o rows not 16-byte aligned) every thread
// stores its row. `done` is this thread's wait on the accumulators; whether to
// go on is decided once for all four warps, so the named barriers are reached
// by all of them or none.
template <int BN>
__device__ __forceinline__ void epilogue_tile(uint32_t tmem, int nacc, int acc_stride, bool done,
                                              const CUtensorMap* omap, bool tma_out, bool split, float* stage,
                                              volatile int* abort_flag, volatile int* go_word, const float* s,
                                              float* o, int out, int tokens, int m0, int n0, int warp, int lane) {
    if (!done) *abort_flag = 1;
    __syncwarp();
    named_bar_sync(1, 128);
    if (warp == 2 && lane == 0) *go_word = *abort_flag ? 0 : 1;
    named_bar_sync(1, 128);
    if (!*go_word) return;
    tc_fence_after();
    const int q = warp & 3;  // this warp's TMEM lane quadrant
    const int m = m0 + q * 32 + lane;
    const float sr = m < out && LQ_IN_BOUNDS(m, out) ? __ldg(s + m) : 0.f;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        float acc[32];
        tmem_ld_32x32b_x32(lane_base + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = __uint_as_float(v[j]);
#pragma unroll 1
        for (int i = 1; i < nacc; ++i) {
            tmem_ld_32x32b_x32(lane_base + i * acc_stride + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] += __uint_as_float(v[j]);
        }
        if (tma_out) {
            // token row c0 + j of the box, this lane's row of W_q at q * 32 + lane:
            // a warp writes 128 consecutive bytes per token
#pragma unroll
            for (int j = 0; j < 32; ++j) stage[(c0 + j) * BM + q * 32 + lane] = sr * acc[j];
        } else if (m < out) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int n = n0 + c0 + j;
                if (n < tokens && LQ_IN_BOUNDS((long long)n * out + m, (long long)tokens * out)) {
                    if (split)
                        atomicAdd(o + (long long)n * out + m, sr * acc[j]);
                    else
                        o[(long long)n * out + m] = sr * acc[j];
                }
            }
        }
    }
    if (tma_out) {
        fence_proxy_async_smem();  // the staged tile, visible to the bulk copy
        named_bar_sync(1, 128);
        if (warp == 2 && lane == 0) {
            if (split)
                tma_reduce_add_2d(omap, smem_addr(stage), m0, n0);
            else
                tma_store_2d(omap, smem_addr(stage), m0, n0);
            bulk_commit_group();
            bulk_wait_group_all();  // complete before the CTA exits and its shared memory is reused
        }
    }
}

template <int BN>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_u, const __grid_constant__ CUtensorMap tmap_o,
                const uint32_t* __restrict__ packed, const float* __restrict__ s, int out, int K, int tokens,
                float* __restrict__ o, int tma_out, unsigned* status) {
    constexpr int B_STAGE = Tile<BN>::B_STAGE, TMEM_COLS = Tile<BN>::TMEM_COLS;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned for the 128-byte swizzle; offsetting the array itself
    // keeps derived pointers in the shared address space
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_STAGE);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* go_word = reinterpret_cast<volatile int*>(tmem_slot + 2);
    const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + STAGES), accf = smem_addr(bars + 2 * STAGES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
    // K split in gridDim.z (1 or 2) parts: this CTA takes k-blocks [kb_lo, kb_hi),
    // the split on a multiple of 8 k-blocks (aligned 16-word groups of sign words)
    const int nkb_all = (K + BK - 1) / BK;
    const int kb_lo = blockIdx.z == 0 ? 0 : (int)((long long)blockIdx.z * nkb_all / gridDim.z) & ~7;
    const int kb_hi = blockIdx.z + 1 == gridDim.z ? nkb_all : (int)((long long)(blockIdx.z + 1) * nkb_all / gridDim.z) & ~7;
    const int nkb = kb_hi - kb_lo;
    const bool split = gridDim.z > 1;

    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(full0 + 8 * st, 1 + UNPACK_THREADS);
            mbar_init(empty0 + 8 * st, 1);
        }
        mbar_init(accf, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmap_u);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                const int st = kb % STAGES, round = kb / STAGES;
                if (round > 0 && !mbar_wait(empty0 + 8 * st, (round - 1) & 1, status)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(full0 + 8 * st, B_STAGE);
                tma_load_2d(smem_addr(sB + st * B_STAGE), &tmap_u, (kb_lo + kb) * BK, n0, full0 + 8 * st);
                issued = kb + 1;
            }
            // Do not leave copies in flight: wait (bounded) for the last load of each stage.
            for (int kb = issued - STAGES < 0 ? 0 : issued - STAGES; kb < issued; ++kb)
                mbar_wait(full0 + 8 * (kb % STAGES), (kb / STAGES) & 1, status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(BM, BN);
            for (int kb = 0; kb < nkb; ++kb) {
                const int st = kb % STAGES, round = kb / STAGES;
                if (!mbar_wait(full0 + 8 * st, round & 1, status)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a_base = smem_addr(sA + st * A_STAGE), b_base = smem_addr(sB + st * B_STAGE);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    umma_f16(tmem, smem_desc_sw128(a_base + kk * 32), smem_desc_sw128(b_base + kk * 32), idesc,
                             (kb | kk) != 0);
                umma_commit(empty0 + 8 * st);
            }
            umma_commit(accf);  // fires once every issued MMA has completed
        }
    } else {
        // ---- unpack: thread `row` writes row `row` of every A stage
        const int row = threadIdx.x - 64;
        const int kw = K >> 5;
        const int grow = m0 + row < out ? m0 + row : out - 1;  // rows past `out` are computed but never stored
        const uint32_t* prow = packed + (long long)grow * kw;
        const uint32_t sw = row & 7;
        const uint32_t row_off = (row >> 3) * 1024 + (row & 7) * 128;
        // The row's sign words arrive 8 k-steps (16 words) at a time, the next
        // group requested before the current one is expanded, so the unpackers
        // do not wait a memory round trip per k-step.
        const bool vec = (kw & 3) == 0;  // 16-byte aligned rows
        auto load16 = [&](int kg0, uint32_t (&w)[16]) {
            if (vec && (kg0 & 1) == 0 && 2 * kg0 + 16 <= kw &&
                LQ_IN_BOUNDS((long long)grow * kw + 2 * kg0 + 15, (long long)out * kw)) {
                const uint4* src = reinterpret_cast<const uint4*>(prow + 2 * kg0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 x = __ldg(src + q);
                    w[4 * q] = x.x;
                    w[4 * q + 1] = x.y;
                    w[4 * q + 2] = x.z;
                    w[4 * q + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q)  // u is zero past K
                    w[q] = 2 * kg0 + q < kw && LQ_IN_BOUNDS((long long)grow * kw + 2 * kg0 + q, (long long)out * kw)
                               ? __ldg(prow + 2 * kg0 + q)
                               : 0u;
            }
        };
        uint32_t cur[16], nxt[16];
        load16(kb_lo, cur);
        bool stop = false;
        for (int kb0 = 0; kb0 < nkb && !stop; kb0 += 8) {
            if (kb0 + 8 < nkb) load16(kb_lo + kb0 + 8, nxt);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int kb = kb0 + kk;
                if (kb >= nkb || stop) break;
                const int st = kb % STAGES, round = kb / STAGES;
                uint32_t v[32];
                expand16(cur[2 * kk] & 0xFFFFu, v);
                expand16(cur[2 * kk] >> 16, v + 8);
                expand16(cur[2 * kk + 1] & 0xFFFFu, v + 16);
                expand16(cur[2 * kk + 1] >> 16, v + 24);
                if (round > 0 && !mbar_wait(empty0 + 8 * st, (round - 1) & 1, status)) {
                    *abort_flag = 1;
                    stop = true;
                    break;
                }
                const uint32_t dst = smem_addr(sA + st * A_STAGE) + row_off;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_shared_v4(dst + ((c ^ sw) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                fence_proxy_async_smem();
                mbar_arrive(full0 + 8 * st);
            }
#pragma unroll
            for (int q = 0; q < 16; ++q) cur[q] = nxt[q];
        }

        // ---- epilogue: TMEM -> registers -> s[r] * acc -> o[t][r], staged in the A / B stages
        static_assert(STAGES * (A_STAGE + B_STAGE) >= BN * BM * 4, "the output tile must fit the operand stages");
        const bool done = mbar_wait(accf, 0, status);
        epilogue_tile<BN>(tmem, 1, 0, done, &tmap_o, tma_out != 0, split, reinterpret_cast<float*>(sA), abort_flag,
                          go_word, s, o, out, tokens, m0, n0, warp, lane);
    }

    // lane 0 of the producer and issuer warps ran its role alone: reconverge
    // every warp before the CTA barrier that orders the TMEM release
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int BN, int NI, int S>
__global__ void __launch_bounds__(TileTA<BN, NI, S>::THREADS, 1)
    gemm_kernel_ta(const __grid_constant__ CUtensorMap tmap_u, const __grid_constant__ CUtensorMap tmap_o,
                const uint32_t* __restrict__ packed, const float* __restrict__ s, int out, int K, int tokens,
                float* __restrict__ o, int tma_out, unsigned* status) {
    constexpr int STAGES = S;  // A stages in TMEM, B stages in shared memory
    constexpr int B_STAGE = Tile<BN>::B_STAGE, TMEM_COLS = TileTA<BN, NI, S>::TMEM_COLS, A_COL = TileTA<BN, NI, S>::A_COL;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned for the 128-byte swizzle; offsetting the array itself
    // keeps derived pointers in the shared address space
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t* sB = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_STAGE);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* go_word = reinterpret_cast<volatile int*>(tmem_slot + 2);
    const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + STAGES), accf = smem_addr(bars + 2 * STAGES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
    // K split in gridDim.z (1 or 2) parts: this CTA takes k-blocks [kb_lo, kb_hi),
    // the split on a multiple of 8 k-blocks (aligned 16-word groups of sign words)
    const int nkb_all = (K + BK - 1) / BK;
    const int kb_lo = blockIdx.z == 0 ? 0 : (int)((long long)blockIdx.z * nkb_all / gridDim.z) & ~7;
    const int kb_hi = blockIdx.z + 1 == gridDim.z ? nkb_all : (int)((long long)(blockIdx.z + 1) * nkb_all / gridDim.z) & ~7;
    const int nkb = kb_hi - kb_lo;
    const bool split = gridDim.z > 1;

    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(full0 + 8 * st, 1 + UNPACK_THREADS);
            mbar_init(empty0 + 8 * st, 1);
        }
        mbar_init(accf, NI);  // one commit per issuer
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmap_u);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                const int st = kb % STAGES, round = kb / STAGES;
                if (round > 0 && !mbar_wait(empty0 + 8 * st, (round - 1) & 1, status)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(full0 + 8 * st, B_STAGE);
                tma_load_2d(smem_addr(sB + st * B_STAGE), &tmap_u, (kb_lo + kb) * BK, n0, full0 + 8 * st);
                issued = kb + 1;
            }
            // Do not leave copies in flight: wait (bounded) for the last load of each stage.
            for (int kb = issued - STAGES < 0 ? 0 : issued - STAGES; kb < issued; ++kb)
                mbar_wait(full0 + 8 * (kb % STAGES), (kb / STAGES) & 1, status);
        }
    } else if (warp == 1 || warp >= 6) {
        // issuer `isr` takes k-steps isr, isr + NI, ... into accumulator columns [isr BN, (isr + 1) BN)
        const int isr = warp == 1 ? 0 : warp - 5;
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(BM, BN), acc = tmem + isr * BN;
            for (int kb = isr; kb < nkb; kb += NI) {
                const int st = kb % STAGES, round = kb / STAGES;
                if (!mbar_wait(full0 + 8 * st, round & 1, status)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a_tmem = tmem + A_COL + st * A_COLS, b_base = smem_addr(sB + st * B_STAGE);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)  // 16 k = 8 TMEM columns of A, 32 bytes of a B row
                    umma_f16_tmem_a(acc, a_tmem + kk * 8, smem_desc_sw128(b_base + kk * 32), idesc,
                                    kb != isr || kk != 0);
                umma_commit(empty0 + 8 * st);
            }
            umma_commit(accf);  // fires once every MMA this thread issued has completed
        }
    } else {
        // ---- unpack: thread `row` writes row `row` of every A stage into TMEM
        // lane `row`; a warp may only reach its own lane quadrant (warp % 4)
        const int row = 32 * (warp & 3) + lane;
        const int kw = K >> 5;
        const int grow = m0 + row < out ? m0 + row : out - 1;  // rows past `out` are computed but never stored
        const uint32_t* prow = packed + (long long)grow * kw;
        const uint32_t a_lane = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + A_COL;
        // The row's sign words arrive 8 k-steps (16 words) at a time, the next
        // group requested before the current one is expanded, so the unpackers
        // do not wait a memory round trip per k-step.
        const bool vec = (kw & 3) == 0;  // 16-byte aligned rows
        auto load16 = [&](int kg0, uint32_t (&w)[16]) {
            if (vec && (kg0 & 1) == 0 && 2 * kg0 + 16 <= kw &&
                LQ_IN_BOUNDS((long long)grow * kw + 2 * kg0 + 15, (long long)out * kw)) {
                const uint4* src = reinterpret_cast<const uint4*>(prow + 2 * kg0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 x = __ldg(src + q);
                    w[4 * q] = x.x;
                    w[4 * q + 1] = x.y;
                    w[4 * q + 2] = x.z;
                    w[4 * q + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q)  // u is zero past K
                    w[q] = 2 * kg0 + q < kw && LQ_IN_BOUNDS((long long)grow * kw + 2 * kg0 + q, (long long)out * kw)
                               ? __ldg(prow + 2 * kg0 + q)
                               : 0u;
            }
        };
        uint32_t cur[16], nxt[16];
        load16(kb_lo, cur);
        // The store of a stage is waited for only after the next k-step has been
        // expanded, so its latency overlaps that work.
        uint32_t v[32];
        bool stop = false;
        int pending = -1;  // stage stored but not yet released to the MMA
        for (int kb0 = 0; kb0 < nkb && !stop; kb0 += 8) {
            if (kb0 + 8 < nkb) load16(kb_lo + kb0 + 8, nxt);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int kb = kb0 + kk;
                if (kb >= nkb || stop) break;
                const int st = kb % STAGES, round = kb / STAGES;
                expand16(cur[2 * kk] & 0xFFFFu, v);
                expand16(cur[2 * kk] >> 16, v + 8);
                expand16(cur[2 * kk + 1] & 0xFFFFu, v + 16);
                expand16(cur[2 * kk + 1] >> 16, v + 24);
                if (pending >= 0) {  // release the previous stage
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(full0 + 8 * pending);
                    pending = -1;
                }
                // tcgen05.st is warp-collective: the warp decides together
                const bool free = round == 0 || mbar_wait(empty0 + 8 * st, (round - 1) & 1, status);
                if (!__all_sync(0xffffffffu, free)) {
                    *abort_flag = 1;
                    stop = true;
                    break;
                }
                // word j holds k-elements (2j, 2j+1): TMEM column j of the stage
                tmem_st_32x32b_x32(a_lane + st * A_COLS, v);
                pending = st;
            }
#pragma unroll
            for (int q = 0; q < 16; ++q) cur[q] = nxt[q];
        }
        if (pending >= 0) {
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(full0 + 8 * pending);
        }

        // ---- epilogue: TMEM -> registers -> s[r] * acc -> o[t][r], staged in the B stages; the
        // issuers' sums are added in issuer order (an issuer without k-steps wrote nothing)
        static_assert(STAGES * B_STAGE >= BN * BM * 4, "the output tile must fit the B stages");
        const bool done = mbar_wait(accf, 0, status);
        epilogue_tile<BN>(tmem, NI < nkb ? NI : nkb, BN, done, &tmap_o, tma_out != 0, split,
                          reinterpret_cast<float*>(sB), abort_flag, go_word, s, o, out, tokens, m0, n0, warp, lane);
    }

    // lane 0 of the producer and issuer warps ran its role alone: reconverge
    // every warp before the CTA barrier that orders the TMEM release
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

template <int BN>
cudaError_t launch_tile(const uint32_t* packed, const float* s, int out, int K, const uint16_t* u_bf16, int tokens,
                        float* o, unsigned* status, cudaStream_t st, int num_sms) {
    EncodeTiledFn encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)tokens};
    cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {BK, BN};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(u_bf16), gdim, gstride, box,
                        estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // o [tokens][out] fp32 for the TMA-store epilogue: rows must be 16-byte aligned
    CUtensorMap omap;
    int tma_out = 0;
    if (out % 4 == 0 && (reinterpret_cast<uintptr_t>(o) & 15u) == 0) {
        cuuint64_t odim[2] = {(cuuint64_t)out, (cuuint64_t)tokens};
        cuuint64_t ostride[1] = {(cuuint64_t)out * 4};
        cuuint32_t obox[2] = {BM, BN};
        tma_out = encode(&omap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, o, odim, ostride, obox, estride,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    if (!tma_out) omap = map;  // unused by the kernel
    // 64-token tiles: A stages in TMEM; wider tiles: A stages in shared memory
    constexpr bool kTA = BN <= 64;
    using TA = TileTA<kTA ? BN : 64, TA_ISSUERS, TA_STAGES>;
    auto kern = [] {
        if constexpr (kTA)
            return gemm_kernel_ta<BN, TA_ISSUERS, TA_STAGES>;
        else
            return gemm_kernel<BN>;
    }();
    constexpr size_t smem = kTA ? TA::SMEM_BYTES : Tile<BN>::SMEM_BYTES;
    constexpr int threads = kTA ? TA::THREADS : THREADS;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    dim3 grid((out + BM - 1) / BM, (tokens + BN - 1) / BN, 1);
    const int nkb = (K + BK - 1) / BK;
    if ((long long)grid.x * grid.y < num_sms && nkb >= 16) {  // too few tiles for the SMs: split K in two
        grid.z = 2;
        cudaError_t e = cudaMemsetAsync(o, 0, (size_t)tokens * out * sizeof(float), st);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, threads, smem, st>>>(map, omap, packed, s, out, K, tokens, o, tma_out, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const uint32_t* packed, const float* s, int out, int K, const uint16_t* u_bf16,
                        int tokens, float* o, unsigned* status, cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // short token runs: 64-token tiles (less idle MMA width and u traffic)
    if (tokens <= 64) return launch_tile<64>(packed, s, out, K, u_bf16, tokens, o, status, st, sms);
    return launch_tile<256>(packed, s, out, K, u_bf16, tokens, o, status, st, sms);
}

}  // namespace lq

LQ_DEBUG_FLAG_TAKE(debug_take_gemm)
