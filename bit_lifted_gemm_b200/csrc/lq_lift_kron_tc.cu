// Prefill lift with a Kronecker-factored whitening on the fifth-generation
// tensor cores (LiftQuant paper note, "Key designs" 3: T = diag(s1) (P1 kron P2)
// diag(s2), so T^{-1} = diag(r2) (Q1 kron Q2) diag(r1); "Key designs" 4: then
// the per-block lift u_blk = M^T a'_blk). With one token's activations read as
// the n1 x n2 matrix X (element i1 * n2 + i2), (Q1 kron Q2) x = Q1 X Q2^T, taken
// as two contractions over all tokens of the call:
//
//   Z[t][i1][j2] = sum_i2 a[t][i1 n2 + i2] * r1[i1 n2 + i2] * Q2[j2][i2]     (kron_z_kernel)
//   a'[t][j1 n2 + j2] = r2[blk] * sum_i1 Q1[j1][i1] * Z[t][i1][j2]           (kron_y_kernel)
//
// followed by the lift of each d-block of a' (CUDA cores, fp32) and bf16 u.
//
// kron_z_kernel: M = 128 tokens, N = n2 (the j2 of one i1), K = i2 (padded to a
// multiple of 64; the padded positions of B are zero). A = the bf16 activations
// themselves, by TMA (128-byte swizzle); B = r1-scaled rows of Q2, which are
// fp32: split into three bf16 parts (hi, mid, lo: 24 significant bits), each a
// B operand accumulating into the same fp32 TMEM tile. One i1 per CTA, whose B
// parts are built once and kept while the CTA runs through its range of token
// tiles (grid: n1 x ranges); two TMEM accumulators, so the epilogue of one tile
// overlaps the MMAs of the next. Z leaves in fp32 by TMA store.
//
// kron_y_kernel: per token, M = j1 (Q1 rows, padded to 128 with zero rows),
// N = j2, K = i1 (n1 <= 64: one 64-wide atom). A = Q1 in three bf16 parts
// (K-major, built once per CTA). B = Z_t: its fp32 [i1][j2] tile comes by TMA,
// and the worker warps split it into three bf16 parts written in the MN-major
// operand layout with the 128-byte swizzle (64 j2 per 128-byte row, eight i1
// rows per 1 KB atom). The six products whose part indices sum to at most two
// keep ~2^-24 relative accuracy, as fp32 arithmetic would (two parts, 16
// significant bits, left elements with cancellation past a bf16 ulp). TMEM
// lane j1 then holds a' for the n2 consecutive channels j1 n2 .. j1 n2 + n2 - 1,
// i.e. whole d-blocks when d divides n2: the same warps apply r2 and the lift
// block by block and store bf16 u, one token behind the parts they produce.
//
// Scratch: Z of token t is written into row t of u itself (fp32, the first
// 4 in bytes of the row), which the lift of token t later overwrites entirely
// (this path needs D >= 2 d, so u has K >= 2 in bf16 columns, and the lifted
// columns [0, in D / d) cover the scratch). The CTA that lifts token t is the
// one that read its Z, so the reads precede the writes.
//
// Every wait is bounded; warps whose lane 0 runs a role alone reconverge before
// the CTA barriers.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "lq_debug.cuh"
#include "lq_internal.h"
#include "lq_sm100.cuh"

namespace lq {
namespace {

using namespace sm100;

constexpr int KZ_TOK = 128;       // tokens per kron_z CTA (MMA M, TMEM lanes)
constexpr int KZ_ASTAGES = 3;     // token tiles of activations in flight
constexpr int KZ_THREADS = 320;   // warp 0 TMA, warp 1 MMA, warps 2..9 B parts, then 2..5 epilogue
constexpr int KZ_PARTS = 3;
constexpr int KY_THREADS = 320;   // warp 0 TMA, warp 1 MMA, warps 2..9 A producers, then epilogue
constexpr int KY_SLOTS = 2;       // tokens in flight (TMEM accumulators)
constexpr int KY_MAXZ = 3;        // fp32 Z tiles in flight (at most)
constexpr uint32_t kSpinK = 1000000000u;

struct KronTcArgs {
    const float* r1;  // [in] or null
    const float* q1;  // [n1][n1]
    const float* q2;  // [n2][n2]
    const float* r2;  // [in / d] or null
    const float* M;   // [d][D]
    __nv_bfloat16* u; // [batch][K]: scratch for Z, then the lifted activations
    unsigned* status;
    int batch, in, n1, n2, d, D, K;
    int n1p, n2p;     // n1 rounded up to 16 (K2's K), n2 rounded up to 16 (N of both)
    int natz;         // 64-element K atoms of kron_z (ceil(n2 / 64))
    int nz;           // fp32 Z tiles in flight in kron_y
    int nza;          // activation tiles in flight in kron_z
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// bf16 part of two values (one packed conversion), the remainders left in
// place (exact in fp32); the last part leaves them alone.
template <bool LAST>
__device__ __forceinline__ uint32_t take_part2(float& x0, float& x1) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const uint32_t w = *reinterpret_cast<const uint32_t*>(&h);
    if (!LAST) {
        x0 -= __uint_as_float(w << 16);
        x1 -= __uint_as_float(w & 0xffff0000u);
    }
    return w;
}

// One part of 64 values into a 128-byte K-major row of a swizzled operand
// (16-byte chunk q at q ^ sw).
template <bool LAST>
__device__ __forceinline__ void store_row_part(float (&x)[64], uint32_t dst, uint32_t sw) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t v0 = take_part2<LAST>(x[8 * q], x[8 * q + 1]);
        const uint32_t v1 = take_part2<LAST>(x[8 * q + 2], x[8 * q + 3]);
        const uint32_t v2 = take_part2<LAST>(x[8 * q + 4], x[8 * q + 5]);
        const uint32_t v3 = take_part2<LAST>(x[8 * q + 6], x[8 * q + 7]);
        st_shared_v4(dst + ((q ^ sw) << 4), v0, v1, v2, v3);
    }
}

__device__ __forceinline__ void named_barrier_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

// Shared -> global tensor copy of a 3-D box (the store completes in the bulk
// group of the issuing thread).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
                 "r"(src), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the bulk stores of this thread have read their shared-memory sources.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until the bulk stores of this thread are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// 64 elements of M or N per 128-byte row, eight K rows per 1 KB atom; lbo =
// bytes between 64-element chunks of M/N, sbo = bytes between 8-row K groups.
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// ============================================================================ Z = X' Q2^T
// One CTA: one i1 and a run of 128-token tiles. The three B parts of i1
// (r1-scaled Q2, zero past n2) are built once and stay; the token tiles of the
// activations stream through a ring; two TMEM accumulators let the epilogue of
// one tile overlap the MMAs of the next.
struct KzLayout {
    uint32_t atomA, atomB, tileA, partB, b, a, zs, bars, total;
};

// nza: activation tiles in flight; zs: the fp32 Z tile [128 tokens][n2] staged
// for its TMA store
__host__ __device__ inline KzLayout kz_layout(int n2p, int natz, int nza) {
    KzLayout L;
    L.atomA = KZ_TOK * 128;                  // 64 K elements of 128 token rows
    L.atomB = (uint32_t)n2p * 128;           // 64 K elements of n2p rows
    L.tileA = natz * L.atomA;
    L.partB = natz * L.atomB;
    L.b = 0;
    L.a = KZ_PARTS * L.partB;                // multiples of 1024 (n2p is a multiple of 16)
    L.zs = L.a + nza * L.tileA;
    L.bars = L.zs + (uint32_t)KZ_TOK * n2p * 4;
    L.total = L.bars + 8 * (2 * KZ_ASTAGES + 4 + 2) + 16;
    return L;
}

__global__ void __launch_bounds__(KZ_THREADS, 1)
    kron_z_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap zsmap,
                  const KronTcArgs p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int natz = p.natz;
    const int nza = p.nza;
    const KzLayout L = kz_layout(p.n2p, natz, nza);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * KZ_ASTAGES + 4 + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t afull0 = smem_addr(bars), aempty0 = afull0 + 8 * KZ_ASTAGES;
    const uint32_t dfull0 = aempty0 + 8 * KZ_ASTAGES, dempty0 = dfull0 + 16;
    const uint32_t bready = dempty0 + 16, mmadone = bready + 8;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i1 = blockIdx.x;
    const int ntiles = (p.batch + KZ_TOK - 1) / KZ_TOK;
    const int tt0 = (int)((long long)blockIdx.y * ntiles / gridDim.y);
    const int tt1 = (int)((long long)(blockIdx.y + 1) * ntiles / gridDim.y);
    const int nt = tt1 - tt0;  // this CTA's token tiles

    if (threadIdx.x == 0) {
        for (int s = 0; s < nza; ++s) {
            mbar_init(afull0 + 8 * s, 1);
            mbar_init(aempty0 + 8 * s, 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(dfull0 + 8 * s, 1);
            mbar_init(dempty0 + 8 * s, 4);  // the four epilogue warps
        }
        mbar_init(bready, 256);
        mbar_init(mmadone, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&amap);
    }
    // the activations are written by the kernel before this one; and no tensor
    // memory is held while waiting for it (a CTA of that kernel may still need
    // tensor memory on this SM)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int k = 0; k < nt; ++k) {
                const int st = k % nza, round = k / nza;
                if (round > 0 && !mbar_wait(aempty0 + 8 * st, (round - 1) & 1, p.status, kSpinK)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(afull0 + 8 * st, L.tileA);
                for (int at = 0; at < natz; ++at)
                    tma_load_2d(smem_addr(smem + L.a + st * L.tileA + at * L.atomA), &amap, i1 * p.n2 + 64 * at,
                                (tt0 + k) * KZ_TOK, afull0 + 8 * st);
                issued = k + 1;
            }
            for (int k = issued > nza ? issued - nza : 0; k < issued; ++k)  // leave no copy in flight
                mbar_wait(afull0 + 8 * (k % nza), (k / nza) & 1, p.status, kSpinK);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(KZ_TOK, p.n2p);
            bool ok = mbar_wait(bready, 0, p.status, kSpinK);
            for (int k = 0; k < nt && ok; ++k) {
                const int st = k % nza, buf = k & 1;
                ok = mbar_wait(afull0 + 8 * st, (k / nza) & 1, p.status, kSpinK);
                if (ok && k >= 2) ok = mbar_wait(dempty0 + 8 * buf, ((k >> 1) - 1) & 1, p.status, kSpinK);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_base = smem_addr(smem + L.a + st * L.tileA), b_base = smem_addr(smem + L.b);
                for (int part = 0; part < KZ_PARTS; ++part)
                    for (int ks = 0; ks < 4 * natz; ++ks)
                        umma_f16(tmem + (uint32_t)(buf * 128),
                                 smem_desc_sw128(a_base + (ks >> 2) * L.atomA + (ks & 3) * 32),
                                 smem_desc_sw128(b_base + part * L.partB + (ks >> 2) * L.atomB + (ks & 3) * 32), idesc,
                                 (part | ks) != 0);
                umma_commit(aempty0 + 8 * st);
                umma_commit(dfull0 + 8 * buf);
            }
            if (!ok) *abort_flag = 1;
            umma_commit(mmadone);
            mbar_wait(mmadone, 0, p.status, kSpinK);
        }
    } else {
        // ---- B parts of i1, once: thread (n, h) owns row n (j2) and K atom h (i2 in [64h, 64h + 64))
        const int w = threadIdx.x - 64;
        const int n = w & 127, h = w >> 7;
        if (n < p.n2p && h < natz) {
            float x[64];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int i2 = 64 * h + 4 * q;
                float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
                if (n < p.n2 && i2 < p.n2) {
                    f = __ldg(reinterpret_cast<const float4*>(p.q2 + (size_t)n * p.n2 + i2));
                    if (p.r1) {
                        const float4 r = __ldg(reinterpret_cast<const float4*>(p.r1 + (size_t)i1 * p.n2 + i2));
                        f.x *= r.x;
                        f.y *= r.y;
                        f.z *= r.z;
                        f.w *= r.w;
                    }
                }
                x[4 * q] = f.x;
                x[4 * q + 1] = f.y;
                x[4 * q + 2] = f.z;
                x[4 * q + 3] = f.w;
            }
            const uint32_t dst = smem_addr(smem + L.b + h * L.atomB) + (n >> 3) * 1024 + (n & 7) * 128;
            store_row_part<false>(x, dst, n & 7);
            store_row_part<false>(x, dst + L.partB, n & 7);
            store_row_part<true>(x, dst + 2 * L.partB, n & 7);
            fence_proxy_async_smem();
        }
        mbar_arrive(bready);

        // ---- epilogue: warps 2..5 (the four TMEM lane quarters) stage Z of their
        // tokens (fp32, row t of the tile = 128-token box) in shared memory; one
        // thread stores the box with TMA (one 3-D box: n2 x 1 x 128 tokens).
        // The four warps decide together whether to go on (they meet at named
        // barriers): warp 2's lane 0 snapshots the abort flag before the first.
        if (warp < 6) {
            const int q = warp & 3;
            float* zs = reinterpret_cast<float*>(smem + L.zs);
            volatile int* snap = abort_flag + 1;
            for (int k = 0; k < nt; ++k) {
                const int buf = k & 1;
                if (!mbar_wait(dfull0 + 8 * buf, (k >> 1) & 1, p.status, kSpinK)) *abort_flag = 1;
                if (warp == 2 && lane == 0) *snap = *abort_flag;
                // (also: the previous tile's store has read the staging buffer: its issuer waited)
                named_barrier_sync(2, 128);
                const bool go = *snap == 0;
                if (go) {
                    tc_fence_after();
                    const uint32_t row = smem_addr(zs + (size_t)(32 * q + lane) * p.n2);
                    for (int c0 = 0; c0 < p.n2; c0 += 16) {
                        uint32_t v[16];
                        tmem_ld_x16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * 128 + c0), v);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            st_shared_v4(row + (uint32_t)(c0 + 4 * j) * 4, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(dempty0 + 8 * buf);
                fence_proxy_async_smem();  // the staged tile is visible to the TMA store
                named_barrier_sync(2, 128);
                if (warp == 2 && lane == 0) {
                    if (go) {
                        tma_store_3d(&zsmap, smem_addr(zs), 0, i1, (tt0 + k) * KZ_TOK);
                        bulk_commit();
                    }
                    bulk_wait_read();
                }
                if (!go) break;  // uniform: every warp read the same snapshot
            }
            if (warp == 2 && lane == 0) bulk_wait_all();  // the stores are complete before the kernel ends
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ============================================================================ a' = r2 o Q1 Z, lift
// The lift of one token from its staged a' rows: thread (bi, e4) computes
// outputs 4 e4 .. 4 e4 + 3 of blocks bi, bi + nbi, ... (block b sits in row
// b / bpr at column (b % bpr) d); those four columns of M are in m. DD: d
// known at compile time (0: generic). Consecutive threads write consecutive
// 8-byte pieces of a u row.
template <int DD>
__device__ __forceinline__ void lift_token(const float* aps, int pitch, int bpr, int bi, int nbi, int nblocks, int e4,
                                           int d, const float (&m)[4][16], const float* r2, __nv_bfloat16* urow,
                                           int D, int K) {
    constexpr int DL = DD ? DD : 16;
    const int dd = DD ? DD : d;
    int j1 = bi / bpr, off = bi - j1 * bpr;
    for (int b = bi; b < nblocks; b += nbi) {
        const float* ar = aps + (size_t)j1 * pitch + off * dd;
        float av[DL];
        if constexpr (DD > 0 && DD % 2 == 0) {
#pragma unroll
            for (int i = 0; i < DD / 2; ++i) {
                const float2 f = *reinterpret_cast<const float2*>(ar + 2 * i);
                av[2 * i] = f.x;
                av[2 * i + 1] = f.y;
            }
        } else {
#pragma unroll
            for (int i = 0; i < DL; ++i) av[i] = i < dd ? ar[i] : 0.f;
        }
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < DL; ++i)
#pragma unroll
            for (int c = 0; c < 4; ++c) s4[c] = fmaf(m[c][i], av[i], s4[c]);
        const float sc = r2 ? __ldg(r2 + b) : 1.f;
        const __nv_bfloat162 h0 = __floats2bfloat162_rn(s4[0] * sc, s4[1] * sc);
        const __nv_bfloat162 h1 = __floats2bfloat162_rn(s4[2] * sc, s4[3] * sc);
        if (LQ_IN_BOUNDS((long long)b * D + 4 * e4 + 3, K))  // within the token's row of u
            *reinterpret_cast<uint2*>(urow + (size_t)b * D + 4 * e4) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
        off += nbi;
        while (off >= bpr) {
            off -= bpr;
            ++j1;
        }
    }
}

// Shared-memory plan of kron_y (offsets from a 1024-byte aligned base): the
// three Q1 parts, a ring of fp32 Z tiles, one set of Z parts, the staged
// a' rows (pitch n2 + 4 floats) and M.
struct KyLayout {
    uint32_t atomA, chunkB, partB, zt, a, zr, parts, aps, ms, bars, total;
    int nchunk, pitch;
};

__host__ __device__ inline KyLayout ky_layout(int n1p, int n2, int d, int D, int nz) {
    KyLayout L;
    L.atomA = 128 * 128;                          // Q1 part: 128 rows (j1) x 64 i1 x bf16
    L.nchunk = (n2 + 63) / 64;
    L.chunkB = (uint32_t)n1p * 128;               // one 64-wide j2 chunk of one part of Z_t
    L.partB = (uint32_t)L.nchunk * L.chunkB;
    L.zt = (((uint32_t)n1p * n2 * 4) + 1023) & ~1023u;
    L.pitch = n2 + 4;
    L.a = 0;
    L.zr = 3 * L.atomA;                           // n1p <= 64: one K atom per part
    L.parts = L.zr + nz * L.zt;
    L.aps = L.parts + 3 * L.partB;
    L.ms = L.aps + (((uint32_t)n1p * L.pitch * 4 + 15) & ~15u);
    L.bars = L.ms + (uint32_t)(((d * D + 3) & ~3) * 4);
    L.total = L.bars + 8 * (2 * KY_MAXZ + 2 + 2 * KY_SLOTS + 2) + 16;  // + TMEM address, abort flag, snapshot
    return L;
}

__global__ void __launch_bounds__(KY_THREADS, 1)
    kron_y_kernel(const __grid_constant__ CUtensorMap zmap, const KronTcArgs p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int nz = p.nz;
    const KyLayout L = ky_layout(p.n1p, p.n2, p.d, p.D, nz);
    float* aps = reinterpret_cast<float*>(smem + L.aps);
    float* Ms = reinterpret_cast<float*>(smem + L.ms);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * KY_MAXZ + 2 + 2 * KY_SLOTS + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    // zfull / zempty: a Z tile landed / was read; pfull / pfree: the Z parts were
    // written / their MMAs are done; dfull / dempty: an accumulator is ready /
    // was read into shared memory
    const uint32_t zfull0 = smem_addr(bars), zempty0 = zfull0 + 8 * KY_MAXZ;
    const uint32_t pfull = zempty0 + 8 * KY_MAXZ, pfree = pfull + 8;
    const uint32_t dfull0 = pfree + 8, dempty0 = dfull0 + 8 * KY_SLOTS;
    const uint32_t aready = dempty0 + 8 * KY_SLOTS, mmadone = aready + 8;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // tokens of this CTA: blockIdx.x, + gridDim.x, ...
    const int ntok = p.batch > (int)blockIdx.x ? (p.batch - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nz; ++s) {
            mbar_init(zfull0 + 8 * s, 1);
            mbar_init(zempty0 + 8 * s, 256);
        }
        mbar_init(pfull, 256);
        mbar_init(pfree, 1);
        for (int s = 0; s < KY_SLOTS; ++s) {
            mbar_init(dfull0 + 8 * s, 1);
            mbar_init(dempty0 + 8 * s, 8);  // the eight worker warps
        }
        mbar_init(aready, 256);
        mbar_init(mmadone, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&zmap);
    }
    // Z is written by kron_z, the kernel before this one; no tensor memory is
    // held while waiting for it (its CTAs may still need tensor memory here)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), 128 * KY_SLOTS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int k = 0; k < ntok; ++k) {
                const int st = k % nz, round = k / nz;
                if (round > 0 && !mbar_wait(zempty0 + 8 * st, (round - 1) & 1, p.status, kSpinK)) {
                    *abort_flag = 1;
                    break;
                }
                const int t = (int)blockIdx.x + k * (int)gridDim.x;
                mbar_arrive_expect_tx(zfull0 + 8 * st, (uint32_t)p.n1p * p.n2 * 4);
                tma_load_3d(smem_addr(smem + L.zr + st * L.zt), &zmap, 0, 0, t, zfull0 + 8 * st);
                issued = k + 1;
            }
            for (int k = issued > nz ? issued - nz : 0; k < issued; ++k)  // leave no copy in flight
                mbar_wait(zfull0 + 8 * (k % nz), (k / nz) & 1, p.status, kSpinK);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // A: Q1 parts, K-major; B: Z_t parts, MN-major (bit 16 of the instruction descriptor)
            const uint32_t idesc = idesc_bf16_f32(128, p.n2p) | (1u << 16);
            bool ok = mbar_wait(aready, 0, p.status, kSpinK);
            for (int k = 0; k < ntok && ok; ++k) {
                const int slot = k % KY_SLOTS;
                ok = mbar_wait(pfull, k & 1, p.status, kSpinK);
                if (ok && k >= KY_SLOTS) ok = mbar_wait(dempty0 + 8 * slot, ((k / KY_SLOTS) - 1) & 1, p.status, kSpinK);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(slot * 128);
                const uint32_t a0 = smem_addr(smem + L.a), b0 = smem_addr(smem + L.parts);
                int first = 1;
                // (A part, B part) with part indices summing to at most 2: hi hi,
                // hi mid, mid hi, hi lo, mid mid, lo hi (~2^-24 relative)
                for (int pr = 0; pr < 6; ++pr) {
                    const int ap = pr == 2 || pr == 4 ? 1 : pr == 5 ? 2 : 0;
                    const int bp = pr == 1 || pr == 4 ? 1 : pr == 3 ? 2 : 0;
                    for (int ks = 0; ks < p.n1p / 16; ++ks) {
                        const uint64_t ad = smem_desc_sw128(a0 + (uint32_t)ap * L.atomA + (uint32_t)ks * 32);
                        const uint64_t bd = smem_desc_sw128_mn(b0 + (uint32_t)bp * L.partB + (uint32_t)ks * 2048,
                                                               L.chunkB, 1024);
                        umma_f16(d, ad, bd, idesc, !first);
                        first = 0;
                    }
                }
                umma_commit(pfree);
                umma_commit(dfull0 + 8 * slot);
            }
            if (!ok) *abort_flag = 1;
            umma_commit(mmadone);
            mbar_wait(mmadone, 0, p.status, kSpinK);
        }
    } else {
        const int w = threadIdx.x - 64;  // 0..255
        // ---- A: Q1 in three parts, rows j1 (zero past n1), K = i1 (one 64-wide atom)
        if (w < 128) {
            const int n = w;
            float x[64];
#pragma unroll
            for (int q = 0; q < 64; ++q) x[q] = (n < p.n1 && q < p.n1) ? __ldg(p.q1 + (size_t)n * p.n1 + q) : 0.f;
            const uint32_t a0 = smem_addr(smem + L.a) + (n >> 3) * 1024 + (n & 7) * 128;
            store_row_part<false>(x, a0, n & 7);
            store_row_part<false>(x, a0 + L.atomA, n & 7);
            store_row_part<true>(x, a0 + 2 * L.atomA, n & 7);
            fence_proxy_async_smem();
        }
        for (int i = w; i < p.d * p.D; i += 256) Ms[i] = __ldg(p.M + i);
        mbar_arrive(aready);
        named_barrier_sync(1, 256);  // M is in shared memory for every worker

        // the lift's thread map: quad ec of D / 4 output quads and block offset bi;
        // M's four columns of the quad stay in registers
        const int nec = p.D / 4, nbi = 256 / nec;
        const int bi = w / nec, ec = w - bi * nec;
        float m4[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 16; ++i) m4[c][i] = (i < p.d && bi < nbi) ? Ms[i * p.D + 4 * ec + c] : 0.f;
        const int bpr = p.n2 / p.d, nblocks = p.in / p.d;
        const int ngr = p.n2 / 8, nitem = p.n1p * ngr;
        const int q = warp & 3, half = (warp - 2) >> 2;  // warps 2..5: half 0, 6..9: half 1

        // parts of token k: 16-byte items (i1 row, 8 consecutive j2) of the MN-major
        // swizzled layout, three parts each
        auto produce = [&](int k) -> bool {
            const int st = k % nz;
            bool ok = mbar_wait(zfull0 + 8 * st, (k / nz) & 1, p.status, kSpinK);
            if (ok && k >= 1) ok = mbar_wait(pfree, (k - 1) & 1, p.status, kSpinK);
            if (ok) {
                const float* zt = reinterpret_cast<const float*>(smem + L.zr + st * L.zt);
                const uint32_t pb = smem_addr(smem + L.parts);
                for (int it = w; it < nitem; it += 256) {
                    const int i1 = it / ngr, g = it - i1 * ngr, j0 = 8 * g;
                    float v[8];
                    const float4 f0 = *reinterpret_cast<const float4*>(zt + (size_t)i1 * p.n2 + j0);
                    const float4 f1 = *reinterpret_cast<const float4*>(zt + (size_t)i1 * p.n2 + j0 + 4);
                    v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w;
                    v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
                    const uint32_t off = (uint32_t)(j0 >> 6) * L.chunkB + (uint32_t)(i1 >> 3) * 1024 +
                                         (uint32_t)(i1 & 7) * 128 + ((((uint32_t)(j0 & 63) >> 3) ^ (uint32_t)(i1 & 7)) << 4);
#pragma unroll
                    for (int part = 0; part < 3; ++part) {
                        uint32_t h[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            h[e] = part == 2 ? take_part2<true>(v[2 * e], v[2 * e + 1])
                                             : take_part2<false>(v[2 * e], v[2 * e + 1]);
                        st_shared_v4(pb + (uint32_t)part * L.partB + off, h[0], h[1], h[2], h[3]);
                    }
                }
                fence_proxy_async_smem();
            }
            mbar_arrive(zempty0 + 8 * st);
            mbar_arrive(pfull);
            return ok;
        };

        // a' of token k: accumulator -> shared rows (lane-owning warps, column
        // chunks split between the two warps of a lane quarter), then the lift
        // by every worker with coalesced stores. The workers meet at named
        // barriers, so whether to go on is decided once for all of them: worker
        // 0 takes a snapshot of the abort flag before the first barrier, and
        // every worker reads that snapshot after it (the next snapshot is taken
        // only after the last barrier of the token).
        volatile int* snap = abort_flag + 1;
        auto epilogue = [&](int k) -> bool {
            const int slot = k % KY_SLOTS;
            if (!mbar_wait(dfull0 + 8 * slot, (k / KY_SLOTS) & 1, p.status, kSpinK)) *abort_flag = 1;
            if (w == 0) *snap = *abort_flag;
            named_barrier_sync(1, 256);
            const bool go = *snap == 0;
            if (go && 32 * q < p.n1) {
                tc_fence_after();
                const int j1 = 32 * q + lane;
                for (int c0 = 16 * half; c0 < p.n2; c0 += 32) {
                    uint32_t v[16];
                    tmem_ld_x16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(slot * 128 + c0), v);
                    tmem_ld_wait();
                    if (j1 < p.n1) {
                        const uint32_t dst = smem_addr(aps + (size_t)j1 * L.pitch + c0);
#pragma unroll
                        for (int j = 0; j < 4; ++j) st_shared_v4(dst + 16 * j, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dempty0 + 8 * slot);
            named_barrier_sync(1, 256);  // a' of token k is in shared memory
            const int t = (int)blockIdx.x + k * (int)gridDim.x;
            __nv_bfloat16* urow = p.u + (size_t)t * p.K;
            const bool row_ok = LQ_IN_BOUNDS(t, p.batch);
            if (go && row_ok && bi < nbi) {
                if (p.d == 8)
                    lift_token<8>(aps, L.pitch, bpr, bi, nbi, nblocks, ec, p.d, m4, p.r2, urow, p.D, p.K);
                else if (p.d == 10)
                    lift_token<10>(aps, L.pitch, bpr, bi, nbi, nblocks, ec, p.d, m4, p.r2, urow, p.D, p.K);
                else if (p.d == 16)
                    lift_token<16>(aps, L.pitch, bpr, bi, nbi, nblocks, ec, p.d, m4, p.r2, urow, p.D, p.K);
                else
                    lift_token<0>(aps, L.pitch, bpr, bi, nbi, nblocks, ec, p.d, m4, p.r2, urow, p.D, p.K);
            }
            // lifted columns past the last block are zero
            if (go && row_ok)
                for (int c = nblocks * p.D + w; c < p.K; c += 256) urow[c] = __float2bfloat16_rn(0.f);
            named_barrier_sync(1, 256);  // every worker is done with a' (and with the snapshot)
            return go;
        };
        // the parts of token k, then a' and the lift of token k - 1 (whose MMAs
        // ran meanwhile); every worker leaves the loop at the same k
        for (int k = 0; k <= ntok; ++k) {
            if (k < ntok && !produce(k)) *abort_flag = 1;
            if (k >= 1 && !epilogue(k - 1)) break;
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128 * KY_SLOTS);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_k() {
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

int round_up(int x, int m) { return (x + m - 1) / m * m; }

size_t kz_smem(int n2p, int natz, int nza) { return 1024 + kz_layout(n2p, natz, nza).total; }

// Deepest activation ring (KZ_ASTAGES or 2) that fits; 0 if none.
int kz_depth(int n2p, int natz) {
    for (int nza = KZ_ASTAGES; nza >= 2; --nza)
        if (kz_smem(n2p, natz, nza) <= 227 * 1024) return nza;
    return 0;
}

size_t ky_smem(int n1p, int n2, int d, int D, int nz) { return 1024 + ky_layout(n1p, n2, d, D, nz).total; }

// Deepest Z ring (3 or 2) that fits; 0 if none.
int ky_depth(int n1p, int n2, int d, int D) {
    for (int nz = KY_MAXZ; nz >= 2; --nz)
        if (ky_smem(n1p, n2, d, D, nz) <= 227 * 1024) return nz;
    return 0;
}

}  // namespace

bool lift_kron_tc_supported(bool a_bf16, bool u_bf16, int batch, int in, int n1, int n2, int d, int D, int K) {
    if (!a_bf16 || !u_bf16 || batch < 64) return false;
    if (n1 < 8 || n1 > 64 || n2 < 16 || n2 > 128 || n2 % 16 != 0 || n1 * n2 != in) return false;
    if (d < 1 || d > 16 || n2 % d != 0 || D < 2 * d || D % 4 != 0 || K < 2 * in) return false;
    const int n1p = round_up(n1, 16), n2p = n2;
    return kz_depth(n2p, (n2 + 63) / 64) > 0 && ky_depth(n1p, n2, d, D) > 0;
}

cudaError_t launch_lift_kron_tc(const uint16_t* a, int batch, int in, const float* r1, const float* q1, int n1,
                                const float* q2, int n2, const float* r2, const float* M, int d, int D, void* u,
                                int K, unsigned* status, cudaStream_t st) {
    EncodeTiledFn encode = encode_fn_k();
    if (!encode) return cudaErrorNotSupported;
    KronTcArgs p;
    p.r1 = r1;
    p.q1 = q1;
    p.q2 = q2;
    p.r2 = r2;
    p.M = M;
    p.u = reinterpret_cast<__nv_bfloat16*>(u);
    p.status = status;
    p.batch = batch;
    p.in = in;
    p.n1 = n1;
    p.n2 = n2;
    p.d = d;
    p.D = D;
    p.K = K;
    p.n1p = round_up(n1, 16);
    p.n2p = n2;
    p.natz = (n2 + 63) / 64;
    p.nz = ky_depth(p.n1p, n2, d, D);
    p.nza = kz_depth(p.n2p, p.natz);
    CUtensorMap amap, zmap, zsmap;
    {  // activations [batch][in] bf16: boxes of 64 channels x 128 tokens
        cuuint64_t gdim[2] = {(cuuint64_t)in, (cuuint64_t)batch};
        cuuint64_t gstride[1] = {(cuuint64_t)in * 2};
        cuuint32_t box[2] = {64, KZ_TOK};
        cuuint32_t es[2] = {1, 1};
        if (encode(&amap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a), gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {  // Z inside u: [token][i1][j2] fp32 (row t of u), one box per token (rows past n1 zero)
        cuuint64_t gdim[3] = {(cuuint64_t)n2, (cuuint64_t)n1, (cuuint64_t)batch};
        cuuint64_t gstride[2] = {(cuuint64_t)n2 * 4, (cuuint64_t)K * 2};
        cuuint32_t box[3] = {(cuuint32_t)n2, (cuuint32_t)p.n1p, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (encode(&zmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, u, gdim, gstride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {  // Z inside u for kron_z's stores: one box of n2 x 1 x 128 tokens (rows past batch are clipped)
        cuuint64_t gdim[3] = {(cuuint64_t)n2, (cuuint64_t)n1, (cuuint64_t)batch};
        cuuint64_t gstride[2] = {(cuuint64_t)n2 * 4, (cuuint64_t)K * 2};
        cuuint32_t box[3] = {(cuuint32_t)n2, 1, KZ_TOK};
        cuuint32_t es[3] = {1, 1, 1};
        if (encode(&zsmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, u, gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const size_t smz = kz_smem(p.n2p, p.natz, p.nza), smy = ky_smem(p.n1p, n2, d, D, p.nz);
    static size_t granted_z[64] = {}, granted_y[64] = {};
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (dev >= 64 || granted_z[dev] < smz) {
        cudaError_t e = cudaFuncSetAttribute(kron_z_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smz);
        if (e != cudaSuccess) return e;
        if (dev < 64) granted_z[dev] = smz;
    }
    if (dev >= 64 || granted_y[dev] < smy) {
        cudaError_t e = cudaFuncSetAttribute(kron_y_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smy);
        if (e != cudaSuccess) return e;
        if (dev < 64) granted_y[dev] = smy;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    // one CTA per (i1, run of token tiles): about one wave of CTAs
    const int ntiles = (batch + KZ_TOK - 1) / KZ_TOK;
    const int runs = std::max(1, std::min(ntiles, sms / n1));  // one wave (one CTA per SM)
    cfg.gridDim = dim3((unsigned)n1, (unsigned)runs, 1);
    cfg.blockDim = dim3(KZ_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smz;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kron_z_kernel, amap, zsmap, p);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)std::min(batch, sms), 1, 1);
    cfg.blockDim = dim3(KY_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smy;
    e = cudaLaunchKernelEx(&cfg, kron_y_kernel, zmap, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace lq

LQ_DEBUG_FLAG_TAKE(debug_take_lift_kron_tc)
