// Quantizer of the tensor-core decode path (lq_decode.h): the lifted
// activations u (fp32 [batch][K]) become the block-scaled 4-bit digit planes
// the tcgen05 contraction reads, once per call, so that no contraction CTA
// repeats the conversion. Every 32-element word is scaled on its own, so there
// is no reduction over K: one warp per word, lane k holding element k. It
// writes seven e2m1 digit planes, per word a delta byte (its exponent below
// the block's largest, and an Inf flag) and, per CTA of kMxQWords words, a
// summary (largest exponent, NaN / Inf, Inf count).
#include "lq_decode.h"
#include "lq_internal.h"

namespace lq {
namespace {

// ------------------------------------------------------------------ block-scaled form

struct QuantMxArgs {
    const float* u;
    uint8_t* planes;   // [kMxPlanes * bpad][K / 2]: row p * bpad + c
    uint8_t* delta;    // [batch][kwp]: per word, its exponent below the CTA's largest (and an Inf flag)
    uint32_t* summ;    // [batch][nqp]: per quantizer CTA
    unsigned* zero;    // group counters of the contraction, cleared here
    int K, kw, kwp, bpad, nq, nqp, nzero;
};

__global__ void __launch_bounds__(32 * kMxQWords) quant_mx_kernel(const QuantMxArgs a) {
    // u is written by the kernel before this one and the workspace may still be
    // read by the previous call's contraction: wait for both, then let the
    // contraction launch (its early reads of the weights thereby also follow
    // whatever preceded this call)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ uint32_t s_sum[kMxQWords];
    const int c = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (blockIdx.x == 0 && c == 0)
        for (int i = threadIdx.x; i < a.nzero; i += blockDim.x) a.zero[i] = 0u;
    const int w = blockIdx.x * kMxQWords + warp;
    uint32_t summ = 0;
    if (w < a.kw) {
        const float x = a.u[(size_t)c * a.K + 32 * w + lane];
        const unsigned bits = __float_as_uint(x) & 0x7fffffffu;
        const unsigned m = __reduce_max_sync(0xffffffffu, bits);
        const bool inf = bits == 0x7f800000u;
        const unsigned ninf = __popc(__ballot_sync(0xffffffffu, inf));
        int d[kMxPlanes];
        uint32_t info;
        if (m > 0x7f800000u) {  // a NaN: the column's output is NaN
            info = kInfoNaN;
#pragma unroll
            for (int p = 0; p < kMxPlanes; ++p) d[p] = 0;
        } else if (m == 0x7f800000u) {  // +-Inf: plane 0 carries their signs (+-1.0), the rest 0
            info = kInfoInf | (ninf << 16);
            d[0] = inf ? (x > 0.f ? 2 : -2) : 0;
#pragma unroll
            for (int p = 1; p < kMxPlanes; ++p) d[p] = 0;
        } else if (m == 0u) {
            info = 0u;
#pragma unroll
            for (int p = 0; p < kMxPlanes; ++p) d[p] = 0;
        } else {
            // max|u| < 2^E (for a subnormal maximum, from its leading bit); q =
            // round(u 2^(20 - E)), |q| <= 2^20, scaled in two exact factors
            const int Ef = (int)(m >> 23);
            const int E = Ef == 0 ? -117 - __clz((int)m) : Ef - 126;
            const int F = 20 - E, Fa = F > 127 ? F / 2 : F;
            const float y = (x * __int_as_float((127 + Fa) << 23)) * __int_as_float((127 + F - Fa) << 23);
            int q = (int)(__float_as_uint(y + 12582912.0f) - 0x4B400000u);  // nearest integer, ties to even
            // balanced base-8 digits, least significant first: d in {-4..3}, top digit in {-4..4}
#pragma unroll
            for (int p = kMxPlanes - 1; p > 0; --p) {
                d[p] = ((q + 4) & 7) - 4;
                q = (q - d[p]) >> 3;
            }
            d[0] = q;
            info = (uint32_t)(E + kMxBias);
        }
        // element k sits at position 8 (k % 4) + k / 4 of the word's 32 nibbles
        // (the order of the sign-word expansion): word k % 4, nibble k / 4
        const int sh = 4 * (lane >> 2);
        uint8_t* dst = a.planes + (size_t)w * 16 + 4 * lane;
#pragma unroll
        for (int p = 0; p < kMxPlanes; ++p) {
            const int dv = d[p];
            uint32_t v = ((uint32_t)(dv < 0 ? 8 - dv : dv)) << sh;  // e2m1 of dv / 2: sign | |dv|
            v |= __shfl_xor_sync(0xffffffffu, v, 4);
            v |= __shfl_xor_sync(0xffffffffu, v, 8);
            v |= __shfl_xor_sync(0xffffffffu, v, 16);
            if (lane < 4) *reinterpret_cast<uint32_t*>(dst + (size_t)(p * a.bpad + c) * (a.K / 2)) = v;
        }
        summ = (info & (kInfoNaN | kInfoInf)) ? (info & (kInfoNaN | kInfoInf)) | (ninf << 16) : info;
    }
    if (lane == 0) s_sum[warp] = summ;
    __syncthreads();
    if (lane == 0) {
        // the CTA's largest exponent over its finite words; each word stores how
        // far below it its own exponent lies (at most 127: further down, its
        // scales underflow to the smallest ue8m0 value whatever the column),
        // bit 7 marking a word that holds +-Inf; all-zero and NaN words store 127
        uint32_t e = 0, f = 0, n = 0;
        for (int i = 0; i < kMxQWords; ++i) {
            const uint32_t v = s_sum[i];
            if (!(v & (kInfoNaN | kInfoInf))) e = max(e, v & kInfoExp);
            f |= v & (kInfoNaN | kInfoInf);
            n += v >> 16;
        }
        if (w < a.kw) {
            const uint32_t v = s_sum[warp];
            uint32_t db = 0x7Fu;
            if (v & kInfoInf)
                db = 0xFFu;
            else if (!(v & kInfoNaN) && (v & kInfoExp) != 0u)
                db = min(127u, e - (v & kInfoExp));
            a.delta[(size_t)c * a.kwp + w] = (uint8_t)db;
        }
        if (warp == 0) a.summ[(size_t)c * a.nqp + blockIdx.x] = e | f | (n << 16);
    }
}

}  // namespace

cudaError_t launch_quant_mx(const float* u, const DecodePlan& p, void* ws, cudaStream_t st) {
    uint8_t* w = static_cast<uint8_t*>(ws);
    QuantMxArgs a;
    a.u = u;
    a.planes = w + p.off_planes;
    a.delta = w + p.off_steps;
    a.summ = reinterpret_cast<uint32_t*>(w + p.off_hdr);
    a.zero = reinterpret_cast<unsigned*>(w + p.off_count);
    a.K = p.K;
    a.kw = p.kw;
    a.bpad = p.tc_bpad;
    a.nq = p.tc_nq;
    a.nqp = p.tc_nqp;
    a.kwp = p.tc_kwp;
    a.nzero = p.tc_groups;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.tc_nq, p.batch, 1);
    cfg.blockDim = dim3(32 * kMxQWords, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, quant_mx_kernel, a);
}

}  // namespace lq
