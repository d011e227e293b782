// Prefill activation lift with the whitening on the fifth-generation tensor
// cores (LiftQuant paper note, "Key designs" 3 and 4: a' = T^{-1} a with a
// block-diagonal T^{-1} of 128 x 128 blocks, then u = blockdiag(M^T) a' per
// block of d channels):
//
//   a'[t][c] = sum_j T^{-1}[c / 128][c % 128][j] a[t][128 (c / 128) + j]
//   u[t][b D + e] = sum_{i < d} M[i][e] a'[t][b d + i]
//
// The whitening is a dense contraction (128 tokens x up to 128 channels x 128
// per block), so it runs as tcgen05.mma kind::f16 with the bf16 activations as
// the A operand. T^{-1} is fp32; to keep fp32 accuracy it is split on the fly
// into three bf16 parts (hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi -
// mid): together 24 significant bits), each a B operand accumulating into the
// same fp32 TMEM tile. The small d -> D lift runs on the CUDA cores in the
// epilogue, which also rounds u to bf16.
//
// One CTA: 128 tokens x one run of G whole lift blocks (G d <= 128 channels,
// so the run touches one or two whitening blocks).
//   warp 0      TMA: the 128 x 128 activation tile of each whitening block
//               (two 64-column boxes, 128-byte swizzle)
//   warp 1      TMEM allocator and single-thread MMA issuer (M 128, N 128, K 16)
//   warps 2..9  split T^{-1} rows into the bf16 parts, stored K-major in the
//               same 128-byte swizzle (row n = channel c0 + n, zero outside the
//               block); warps 2..5 then stage a' from TMEM in shared memory
//   all warps   the lift: a thread keeps its d x W entries of M in registers and
//               walks token rows, consecutive threads on consecutive W-output
//               chunks of a u row (coalesced stores)
// A 2-stage ring of B parts and a single A tile are coupled by mbarriers;
// every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "lq_debug.cuh"
#include "lq_internal.h"
#include "lq_sm100.cuh"

namespace lq {
namespace {

using namespace sm100;

constexpr int TC_TOK = 128;                 // tokens per CTA (MMA M, TMEM lanes)
constexpr int TC_N = 128;                   // accumulator columns = channels of the run (MMA N)
constexpr int TC_BLK = 128;                 // whitening block width (MMA K per block)
constexpr int TC_ATOM = TC_TOK * 64 * 2;    // 128 rows x 64 bf16 (one swizzle span): 16 KB
constexpr int TC_TILE = 2 * TC_ATOM;        // 128 rows x 128 bf16: 32 KB
constexpr int TC_BSTAGES = 2;
constexpr int TC_PARTS = 3;
constexpr int TC_THREADS = 320;
constexpr int TC_WORKERS = 256;             // warps 2..9
constexpr int TC_APITCH = 129;              // staged a' row (floats; odd: conflict-free column reads)
constexpr size_t TC_SMEM_CORE = (size_t)TC_TILE * (1 + TC_BSTAGES);

struct TcArgs {
    const float* tinv;
    const float* M;
    void* u;
    int u_bf16;
    int batch, in, d, D, K, G;
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// bf16 part of two values (one packed conversion), the remainders left in
// place (exact in fp32); the last part leaves them alone.
template <bool LAST>
__device__ __forceinline__ uint32_t take_part(float& x0, float& x1) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);  // x0 in the low half
    const uint32_t w = *reinterpret_cast<const uint32_t*>(&h);
    if (!LAST) {
        x0 -= __uint_as_float(w << 16);
        x1 -= __uint_as_float(w & 0xffff0000u);
    }
    return w;
}

// One part of a producer's 64 values into its row of a B stage.
template <bool LAST>
__device__ __forceinline__ void store_part(float (&x)[64], uint32_t dst, uint32_t sw) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t v0 = take_part<LAST>(x[8 * q], x[8 * q + 1]);
        const uint32_t v1 = take_part<LAST>(x[8 * q + 2], x[8 * q + 3]);
        const uint32_t v2 = take_part<LAST>(x[8 * q + 4], x[8 * q + 5]);
        const uint32_t v3 = take_part<LAST>(x[8 * q + 6], x[8 * q + 7]);
        st_shared_v4(dst + ((q ^ sw) << 4), v0, v1, v2, v3);
    }
}

constexpr int TC_LIFT_MAXD = 16;  // lift blocks up to this size keep a' in registers

// W consecutive outputs u[e0 .. e0 + W) of one (token, lift block) from the d
// values of a' at ar: M rows read from shared memory in float4 vectors where W
// allows, one store of W values.
template <int W, bool REG>
__device__ __forceinline__ void lift_chunk(const float* ar, const float* Ms, const TcArgs& p, int e0, long long uidx) {
    float acc[W];
#pragma unroll
    for (int j = 0; j < W; ++j) acc[j] = 0.f;
    if (REG) {
        float av[TC_LIFT_MAXD];
#pragma unroll
        for (int i = 0; i < TC_LIFT_MAXD; ++i) av[i] = i < p.d ? ar[i] : 0.f;
#pragma unroll
        for (int i = 0; i < TC_LIFT_MAXD; ++i) {
            if (i < p.d) {
                const float* mr = Ms + i * p.D + e0;
                if (W % 4 == 0) {
#pragma unroll
                    for (int v = 0; v < W / 4; ++v) {
                        const float4 m = reinterpret_cast<const float4*>(mr)[v];
                        acc[(4 * v) % W] = fmaf(m.x, av[i], acc[(4 * v) % W]);
                        acc[(4 * v + 1) % W] = fmaf(m.y, av[i], acc[(4 * v + 1) % W]);
                        acc[(4 * v + 2) % W] = fmaf(m.z, av[i], acc[(4 * v + 2) % W]);
                        acc[(4 * v + 3) % W] = fmaf(m.w, av[i], acc[(4 * v + 3) % W]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < W; ++j) acc[j] = fmaf(mr[j], av[i], acc[j]);
                }
            }
        }
    } else {
        for (int i = 0; i < p.d; ++i) {
            const float av = ar[i];
            const float* mr = Ms + i * p.D + e0;
#pragma unroll
            for (int j = 0; j < W; ++j) acc[j] = fmaf(mr[j], av, acc[j]);
        }
    }
    if (!LQ_IN_BOUNDS(uidx + W - 1, (long long)p.batch * p.K)) return;
    if (p.u_bf16) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.u) + uidx;
        if (W == 8) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(acc[(2 * j) % W], acc[(2 * j + 1) % W]);
                w[j] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        } else if (W == 4) {
            const __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[0], acc[1 % W]);
            const __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[2 % W], acc[3 % W]);
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
        } else {
#pragma unroll
            for (int j = 0; j < W; ++j) dst[j] = __float2bfloat16_rn(acc[j]);
        }
    } else {
        float* dst = reinterpret_cast<float*>(p.u) + uidx;
        if (W % 4 == 0) {
#pragma unroll
            for (int v = 0; v < W / 4; ++v)
                reinterpret_cast<float4*>(dst)[v] = make_float4(acc[(4 * v) % W], acc[(4 * v + 1) % W],
                                                                acc[(4 * v + 2) % W], acc[(4 * v + 3) % W]);
        } else {
#pragma unroll
            for (int j = 0; j < W; ++j) dst[j] = acc[j];
        }
    }
}

// The lift of the CTA's tile: items (token, chunk of W outputs) in u-row order,
// consecutive threads on consecutive chunks, so a warp's stores cover
// contiguous stretches of a u row. Generic form (M read from shared memory).
template <int W, bool REG>
__device__ __forceinline__ void lift_tile(const float* aps, const float* Ms, const TcArgs& p, int t0, int b0, int ng,
                                          int w) {
    const int per_blk = p.D / W;                 // chunks per lift block
    const int nch = ng * per_blk;                // chunks per token row of the run
    const int total = TC_TOK * nch;
    const unsigned rb = 0xffffffffu / (unsigned)per_blk;  // quotient estimates, corrected once
    int tok = w / nch, c = w - tok * nch;
    const int dq = TC_WORKERS / nch, dr = TC_WORKERS - dq * nch;
    for (int it = w; it < total; it += TC_WORKERS) {
        if (t0 + tok >= p.batch) break;  // items are token-major: the rest are past the batch too
        int g = (int)__umulhi((unsigned)c, rb);
        if ((g + 1) * per_blk <= c) ++g;
        const int e0 = (c - g * per_blk) * W;
        lift_chunk<W, REG>(aps + tok * TC_APITCH + g * p.d, Ms, p, e0,
                           (long long)(t0 + tok) * p.K + (long long)(b0 + g) * p.D + e0);
        c += dr;
        tok += dq;
        if (c >= nch) {
            c -= nch;
            ++tok;
        }
    }
}

// Loads from shared memory spelled out, so the compiler need not order them
// after the global stores of u (they cannot alias).
__device__ __forceinline__ float lds_f32(const float* q) {
    float v;
    asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(smem_addr(q)));
    return v;
}
__device__ __forceinline__ float4 lds_f32x4(const float* q) {
    float4 v;
    asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(smem_addr(q)));
    return v;
}

// Fast form for lift blocks of DD channels (compile-time) and D % W == 0:
// thread w owns the W-output chunk c = w % nch of the run's row (its DD x W
// entries of M in registers) and walks the tokens w / nch, w / nch + s, ...
// with s = nthreads / nch, two rows per iteration (independent FMA chains);
// per token it reads the block's DD values of a' and does DD W FMAs.
// Consecutive threads write consecutive W-output chunks of a u row.
template <int W, int DD>
__device__ __forceinline__ void lift_tile_fixed(const float* aps, const float* Ms, const TcArgs& p, int t0, int b0,
                                                int ng, int w, int nthreads) {
    const int per_blk = p.D / W;
    const int nch = ng * per_blk;
    const int s = nthreads / nch;  // token rows walked at once
    if (w >= s * nch) return;
    const int c = w % nch, g = c / per_blk, e0 = (c - g * per_blk) * W;
    float m[DD][W];
#pragma unroll
    for (int i = 0; i < DD; ++i) {
        if (W == 4) {
            const float4 v = lds_f32x4(Ms + i * p.D + e0);
            m[i][0] = v.x;
            m[i][1 % W] = v.y;
            m[i][2 % W] = v.z;
            m[i][3 % W] = v.w;
        } else {
#pragma unroll
            for (int j = 0; j < W; ++j) m[i][j] = lds_f32(Ms + i * p.D + e0 + j);
        }
    }
    const int tend = min(TC_TOK, p.batch - t0);
    int tok = w / nch;
    const float* at = aps + tok * TC_APITCH + g * p.d;
    const size_t col = (size_t)(b0 + g) * p.D + e0;
    const size_t rstep = (size_t)s * p.K;  // elements between the two rows of an iteration
    size_t ui = (size_t)(t0 + tok) * p.K + col;
    for (; tok < tend; tok += 2 * s, at += 2 * s * TC_APITCH, ui += 2 * rstep) {
        const bool two = tok + s < tend;
        const float* at2 = two ? at + s * TC_APITCH : at;
        float acc[2][W];
#pragma unroll
        for (int j = 0; j < W; ++j) acc[0][j] = acc[1][j] = 0.f;
#pragma unroll
        for (int i = 0; i < DD; ++i) {
            const float av = lds_f32(at + i), av2 = lds_f32(at2 + i);
#pragma unroll
            for (int j = 0; j < W; ++j) {
                acc[0][j] = fmaf(m[i][j], av, acc[0][j]);
                acc[1][j] = fmaf(m[i][j], av2, acc[1][j]);
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            if (r == 1 && !two) break;
            const size_t uo = ui + (r ? rstep : 0);
            if (!LQ_IN_BOUNDS(uo + W - 1, (long long)p.batch * p.K)) continue;
            if (p.u_bf16) {
                __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.u) + uo;
                if (W == 4) {
                    const __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[r][0], acc[r][1 % W]);
                    const __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[r][2 % W], acc[r][3 % W]);
                    *reinterpret_cast<uint2*>(dst) = make_uint2(*reinterpret_cast<const uint32_t*>(&h0),
                                                                *reinterpret_cast<const uint32_t*>(&h1));
                } else if (W == 2) {
                    *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(acc[r][0], acc[r][1 % W]);
                } else {
                    *dst = __float2bfloat16_rn(acc[r][0]);
                }
            } else {
                float* dst = reinterpret_cast<float*>(p.u) + uo;
                if (W == 4)
                    *reinterpret_cast<float4*>(dst) =
                        make_float4(acc[r][0], acc[r][1 % W], acc[r][2 % W], acc[r][3 % W]);
                else if (W == 2)
                    *reinterpret_cast<float2*>(dst) = make_float2(acc[r][0], acc[r][1 % W]);
                else
                    *dst = acc[r][0];
            }
        }
    }
}

// The fast form for this shape, if there is one (false: use the generic form).
__device__ __forceinline__ bool lift_tile_fast(const float* aps, const float* Ms, const TcArgs& p, int t0, int b0,
                                               int ng, int w, int nthreads) {
    const int W = (p.D & 3) == 0 ? 4 : (p.D & 1) == 0 ? 2 : 1;
    if (nthreads / (ng * (p.D / W)) == 0) return false;  // rows wider than the threads
    if (p.d == 8) {
        if (W == 4) lift_tile_fixed<4, 8>(aps, Ms, p, t0, b0, ng, w, nthreads);
        else if (W == 2) lift_tile_fixed<2, 8>(aps, Ms, p, t0, b0, ng, w, nthreads);
        else lift_tile_fixed<1, 8>(aps, Ms, p, t0, b0, ng, w, nthreads);
        return true;
    }
    if (p.d == 10) {
        if (W == 4) lift_tile_fixed<4, 10>(aps, Ms, p, t0, b0, ng, w, nthreads);
        else if (W == 2) lift_tile_fixed<2, 10>(aps, Ms, p, t0, b0, ng, w, nthreads);
        else lift_tile_fixed<1, 10>(aps, Ms, p, t0, b0, ng, w, nthreads);
        return true;
    }
    return false;
}

__global__ void __launch_bounds__(TC_THREADS, 2)
    lift_tc_kernel(const __grid_constant__ CUtensorMap amap, const TcArgs p, unsigned* status) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned for the 128-byte swizzle; offsetting the array itself
    // keeps derived pointers in the shared address space
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = smem + TC_TILE;
    float* aps = reinterpret_cast<float*>(smem);  // staged a' [128][TC_APITCH], after the MMAs
    float* Ms = reinterpret_cast<float*>(smem + TC_SMEM_CORE);
    const int mpad = (p.d * p.D + 3) & ~3;
    uint64_t* bars = reinterpret_cast<uint64_t*>(Ms + mpad);  // afull, aempty, bfull[2], bempty[2], accf
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t afull = smem_addr(bars), aempty = smem_addr(bars + 1);
    const uint32_t bfull0 = smem_addr(bars + 2), bempty0 = smem_addr(bars + 4), accf = smem_addr(bars + 6);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblocks = p.in / p.d;
    const int b0 = blockIdx.x * p.G, b1 = min(nblocks, b0 + p.G);
    const int ng = b1 - b0;
    const int c0 = b0 * p.d, C = ng * p.d;
    const int t0 = blockIdx.y * TC_TOK;
    const int kb0 = c0 / TC_BLK;
    const int nkb = (c0 + C - 1) / TC_BLK - kb0 + 1;  // whitening blocks touched: 1 or 2
    const int nst = TC_PARTS * nkb;                     // (block, part) operand stages

    if (threadIdx.x == 0) {
        mbar_init(afull, 1);
        mbar_init(aempty, 1);
        for (int s = 0; s < TC_BSTAGES; ++s) {
            mbar_init(bfull0 + 8 * s, TC_WORKERS);
            mbar_init(bempty0 + 8 * s, 1);
        }
        mbar_init(accf, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&amap);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), TC_N);
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
                if (kb > 0 && !mbar_wait(aempty, (kb - 1) & 1, status)) {
                    *abort_flag = 1;
                    break;
                }
                const int x = (kb0 + kb) * TC_BLK;
                mbar_arrive_expect_tx(afull, TC_TILE);
                tma_load_2d(smem_addr(sA), &amap, x, t0, afull);
                tma_load_2d(smem_addr(sA + TC_ATOM), &amap, x + 64, t0, afull);
                issued = kb + 1;
            }
            if (issued > 0) mbar_wait(afull, (issued - 1) & 1, status);  // leave no copy in flight
        } else {
            // M is needed only by the lift at the end: its load stays off the
            // critical path (the barrier before the epilogue orders it)
            for (int i = lane - 1; i < p.d * p.D; i += 31) Ms[i] = __ldg(p.M + i);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(TC_TOK, TC_N);
            for (int idx = 0; idx < nst; ++idx) {
                const int kb = idx / TC_PARTS, part = idx % TC_PARTS;
                const int st = idx % TC_BSTAGES, round = idx / TC_BSTAGES;
                if (part == 0 && !mbar_wait(afull, kb & 1, status)) {
                    *abort_flag = 1;
                    break;
                }
                if (!mbar_wait(bfull0 + 8 * st, round & 1, status)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a_base = smem_addr(sA), b_base = smem_addr(sB + st * TC_TILE);
#pragma unroll
                for (int ks = 0; ks < TC_BLK / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * TC_ATOM + (ks & 3) * 32;
                    umma_f16(tmem, smem_desc_sw128(a_base + off), smem_desc_sw128(b_base + off), idesc,
                             (idx | ks) != 0);
                }
                umma_commit(bempty0 + 8 * st);
                if (part == TC_PARTS - 1) umma_commit(aempty);
            }
            umma_commit(accf);  // fires once every issued MMA has completed
        }
    } else {
        // ---- B operands: thread (n, h) owns row n (channel c0 + n), columns [64h, 64h + 64)
        const int w = threadIdx.x - 64;
        const int n = w & (TC_N - 1), h = w >> 7;
        const uint32_t row_off = (n >> 3) * 1024 + (n & 7) * 128;
        const uint32_t sw = n & 7;
        bool stop = false;
        for (int kb = 0; kb < nkb && !stop; ++kb) {
            const int cb = c0 + n - (kb0 + kb) * TC_BLK;  // row of the channel inside this whitening block
            const bool inb = n < C && cb >= 0 && cb < TC_BLK;
            float x[64];
            if (inb) {
                const float4* src =
                    reinterpret_cast<const float4*>(p.tinv + ((size_t)(kb0 + kb) * TC_BLK + cb) * TC_BLK + 64 * h);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const float4 f = __ldg(src + q);
                    x[4 * q] = f.x;
                    x[4 * q + 1] = f.y;
                    x[4 * q + 2] = f.z;
                    x[4 * q + 3] = f.w;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 64; ++q) x[q] = 0.f;
            }
#pragma unroll
            for (int part = 0; part < TC_PARTS; ++part) {
                const int idx = TC_PARTS * kb + part, st = idx % TC_BSTAGES, round = idx / TC_BSTAGES;
                if (round > 0 && !mbar_wait(bempty0 + 8 * st, (round - 1) & 1, status)) {
                    *abort_flag = 1;
                    stop = true;
                    break;
                }
                const uint32_t dst = smem_addr(sB + st * TC_TILE + h * TC_ATOM) + row_off;
                if (part == TC_PARTS - 1)
                    store_part<true>(x, dst, sw);
                else
                    store_part<false>(x, dst, sw);
                fence_proxy_async_smem();
                mbar_arrive(bfull0 + 8 * st);
            }
        }

    }

    // ---- epilogue, every warp: a' from TMEM into shared memory, then the lift
    const bool done = mbar_wait(accf, 0, status);
    tc_fence_after();
    if (warp >= 2 && warp < 6) {  // warps 2..5 cover the four TMEM lane quadrants
        const int q = warp & 3;
        // tcgen05.ld is warp-collective: decide for the whole warp at once
        if (__all_sync(0xffffffffu, done && !*abort_flag)) {
            float* row = aps + (q * 32 + lane) * TC_APITCH;
            for (int cc = 0; cc < (C + 31) / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + cc * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) row[cc * 32 + j] = __uint_as_float(v[j]);
            }
        }
    }
    __syncwarp();  // reconverge the producer and issuer warps before the CTA barrier
    __syncthreads();
    if (done && !*abort_flag) {
        const int tid = threadIdx.x, w = tid - 64;  // the generic forms use warps 2..9
        if (!lift_tile_fast(aps, Ms, p, t0, b0, ng, tid, TC_THREADS) && w >= 0) {
            if (p.d <= TC_LIFT_MAXD && (p.D & 7) == 0)
                lift_tile<8, true>(aps, Ms, p, t0, b0, ng, w);
            else if (p.d <= TC_LIFT_MAXD && (p.D & 3) == 0)
                lift_tile<4, true>(aps, Ms, p, t0, b0, ng, w);
            else if (p.d <= TC_LIFT_MAXD)
                lift_tile<1, true>(aps, Ms, p, t0, b0, ng, w);
            else
                lift_tile<1, false>(aps, Ms, p, t0, b0, ng, w);
        }
        // lifted entries past nblocks * D are zero; the CTA with the last run writes them
        if (b1 == nblocks) {
            const int tail = p.K - nblocks * p.D;
            for (int it = tid; it < TC_TOK * tail; it += TC_THREADS) {
                const int tok = it / tail, e = it - tok * tail;
                if (t0 + tok >= p.batch) break;
                const long long idx = (long long)(t0 + tok) * p.K + (long long)nblocks * p.D + e;
                if (!LQ_IN_BOUNDS(idx, (long long)p.batch * p.K)) continue;
                if (p.u_bf16)
                    reinterpret_cast<__nv_bfloat16*>(p.u)[idx] = __float2bfloat16_rn(0.f);
                else
                    reinterpret_cast<float*>(p.u)[idx] = 0.f;
            }
        }
    }

    // lane 0 of the producer and issuer warps ran its role alone: reconverge
    // every warp before the CTA barrier that orders the TMEM release
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TC_N);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* q = nullptr;
        cudaDriverEntryPointQueryResult r;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &r) == cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(q);
    }
    return fn;
}

size_t tc_smem(int d, int D) {
    return 1024 /*alignment slack*/ + TC_SMEM_CORE + sizeof(float) * (size_t)((d * D + 3) & ~3) + 7 * 8 + 16;
}

}  // namespace

bool lift_tc_supported(bool a_bf16, int batch, int in, const float* tinv, int tblk, int d, int D) {
    return a_bf16 && tinv && tblk == TC_BLK && batch >= TC_TOK / 2 && in % TC_BLK == 0 && d <= TC_N &&
           in % d == 0 && tc_smem(d, D) <= 113 * 1024;
}

cudaError_t launch_lift_tc(const uint16_t* a, int batch, int in, const float* tinv, const float* M, int d, int D,
                           void* u, bool u_bf16, int K, unsigned* status, cudaStream_t st) {
    EncodeTiledFn encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    cuuint64_t gdim[2] = {(cuuint64_t)in, (cuuint64_t)batch};
    cuuint64_t gstride[1] = {(cuuint64_t)in * 2};
    cuuint32_t box[2] = {64, TC_TOK};
    cuuint32_t estride[2] = {1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    TcArgs p;
    p.tinv = tinv;
    p.M = M;
    p.u = u;
    p.u_bf16 = u_bf16;
    p.batch = batch;
    p.in = in;
    p.d = d;
    p.D = D;
    p.K = K;
    p.G = TC_N / d;
    const int nblocks = in / d;
    const size_t smem = tc_smem(d, D);
    static size_t granted[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || granted[dev] < smem) {
        cudaError_t e = cudaFuncSetAttribute(lift_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) granted[dev] = smem;
    }
    const dim3 grid((nblocks + p.G - 1) / p.G, (batch + TC_TOK - 1) / TC_TOK);
    lift_tc_kernel<<<grid, TC_THREADS, smem, st>>>(map, p, status);
    return cudaGetLastError();
}

}  // namespace lq

LQ_DEBUG_FLAG_TAKE(debug_take_lift_tc)
