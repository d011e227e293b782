// Decode-path plan and workspace layout, shared by the quantizer of the
// tensor-core path (lq_quant.cu), the two decode contraction kernels
// (lq_gemv.cu on mma.sync, lq_gemv_tc.cu on tcgen05) and the C ABI (lq_api.cu).
//
// mma.sync path (up to three columns): each CTA quantizes the K range of its
// launch itself, column by column, to 32-bit fixed point with one
// power-of-two scale, u_q[c][k] = round(u[c][k] * 2^F_c), |u_q| <= 2^30, held
// as four balanced int8 digit planes u_q = d0 + 2^8 d1 + 2^16 d2 + 2^24 d3 (the
// bytes of (u_q + 0x80808080) ^ 0x80808080). An element's rounding error is at
// most 2^-31 of the largest |u| of its column and K range. The kernel adds the
// digits of the set bits exactly in integers (sum sigma u_q = 2 sum_{bit=1} u_q
// - sum u_q), so the only rounding is this quantization and the final stores.
// Columns holding a NaN are written as NaN; columns holding +-Inf are
// contracted on their Inf pattern (lq_gemv.cu).
//
// tcgen05 path (four or more columns): the block-scaled 4-bit form below,
// quantized once per call into the workspace.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace lq {

constexpr int kPlanes = 4;       // int8 digit planes of the 32-bit fixed point
constexpr int kStepWords = 16;   // words of K per weight step of the mma.sync kernel
constexpr int kMaxColsPass = 2;  // batch columns per mma.sync pass (8 digit columns = one n8 tile)

enum : int { kColFinite = 0, kColInf = 1, kColNaN = 2 };

// 16-byte chunk index of word pair (x, x+1), x even, in an mma.sync digit
// plane: the four chunks from 2x + x/4 (the x/4 skew keeps a quarter-warp's
// 16-byte loads on distinct banks).
__host__ __device__ inline int chunkpos(int x) { return 2 * x + (x >> 2); }

// Chunks per mma.sync plane for `words` words: covers chunkpos(words - 1) + 4
// and is 4 (mod 8), which separates the planes a quarter-warp reads.
__host__ __device__ inline int plane_pitch(int words) {
    int cp = 2 * words + words / 4 + 4;
    return cp % 8 == 4 ? cp : cp + 4;
}

// ---- block-scaled 4-bit form (the tcgen05 kind::mxf4 kernel, lq_gemv_tc.cu)
//
// Each 32-element word w of a column is scaled on its own: with E the exponent
// of its largest |u| (max|u| < 2^E), q = round(u * 2^(20 - E)) (|q| <= 2^20) is
// written in kMxPlanes balanced base-8 digits d_p in {-4..4}, most significant
// first, so u ~ sum_p d_p 2^(E - 2 - 3p) (error <= 2^(E - 21)). Digit p of
// element k is the e2m1 value d_p / 2 (exact: 0, +-0.5 .. +-2). The B operand
// of the MMA is then plane p of column c with the per-word scale factor
// 2^(E - 1 - 3p - G_c), G_c being the column's largest E, which the kernel
// applies through the ue8m0 block scales (normalized so the accumulators stay
// near 1) and undoes in its epilogue.
constexpr int kMxPlanes = 7;
constexpr int kMxQWords = 8;  // words of one column per quantizer CTA (one per warp)

// A word's info (inside the quantizer): bits 0..8 the biased exponent E + kMxBias
// (0: the word is all zero; E runs from -148 for the smallest subnormal to 128),
// bit 9 a NaN in the word, bit 10 an Inf, bits 16..21 the number of +-Inf
// elements. Per quantizer CTA (kMxQWords words of one column) the workspace keeps
// a summary: bits 0..8 the largest biased exponent E_loc of its finite words,
// bit 9 any NaN, bit 10 any Inf, bits 16..31 the number of +-Inf elements; and
// per word one delta byte: min(127, E_loc - E) (127 for all-zero and NaN
// words), bit 7 set for a word holding +-Inf. The contraction rebuilds each
// scale exponent from them with byte-wise saturating arithmetic.
constexpr int kMxBias = 150;
constexpr uint32_t kInfoExp = 0x1ffu, kInfoNaN = 1u << 9, kInfoInf = 1u << 10;

// Launch plan of one decode contraction and the layout of its workspace.
struct DecodePlan {
    int out, K, kw, batch;
    bool tc;  // block-scaled tcgen05 kernel (else mma.sync on 32-bit fixed point)

    // ---- mma.sync kernel (lq_gemv.cu)
    int grid, ts, stages, cols, npass, kwc, nchunk, pitch, maxgroups;
    bool tma, ustage;  // weights through TMA rings; u staged by TMA (else read directly)
    size_t smem;
    size_t image_bytes;  // shared-memory digit planes of one (pass, K chunk): kPlanes * cols * pitch * 16

    // ---- tcgen05 kernel (lq_gemv_tc.cu)
    int tc_grid, tc_bpad, tc_n, tc_groups, tc_stages, tc_maxcontrib, tc_nq, tc_nacc, tc_nss, tc_nsa, tc_mt;
    int tc_nqp, tc_kwp;     // pitches of the summaries (multiple of 4) and word deltas (of 16)
    long long tc_units;     // (row group, K stage) units over all groups
    size_t tc_smem;
    size_t row_bytes;       // bytes of one B row (one plane of one column): K / 2

    // ---- workspace (byte offsets from its 256-byte aligned base)
    //   mma.sync: none used (256 bytes are still asked for)
    //   tcgen05:  hdr = column summaries uint32 [batch][tc_nqp], steps = word deltas
    //             uint8 [batch][tc_kwp], planes = B rows [kMxPlanes * tc_bpad][K / 2] (row p * tc_bpad + c),
    //             count = group counters, slots = split partial sums
    size_t off_hdr, off_steps, off_planes, off_count, off_slots, bytes;
};

// Host: the plan for (out, K, batch); .bytes == 0 if no plan fits.
DecodePlan make_decode_plan(int out, int K, int batch);

}  // namespace lq
