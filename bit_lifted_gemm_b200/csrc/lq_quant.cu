// Decode-path quantizers (lq_decode.h): the lifted activations u (fp32
// [batch][K]) become the digit planes the contraction kernel reads, once per
// call, so that no contraction CTA repeats the conversion.
//
// quant_kernel (for the mma.sync kernel): each column becomes 32-bit fixed point
// with one power-of-two scale, as four balanced int8 digit planes, plus per-step
// sums of u_q and Inf counts and a per-column header. One CTA per column, 1024
// threads. Pass 1 takes the largest |u| (its float bits also reveal NaN and
// Inf); pass 2 converts. A thread handles items (word x, position j): elements
// j, j + 8, j + 16, j + 24 of word x, which become one 32-bit digit register per
// plane. A warp's 32 items are four words of one 16-word step, so step sums
// need one shared atomic per warp.
//
// quant_mx_kernel (for the tcgen05 kernel): every 32-element word is scaled on
// its own, so there is no reduction over K: one warp per word, lane k holding
// element k. It writes seven e2m1 digit planes, the word's info word and, per
// CTA, a column summary (largest exponent, NaN / Inf, Inf count).
#include "lq_decode.h"
#include "lq_internal.h"

namespace lq {
namespace {

constexpr int kQThreads = 1024;
constexpr int kQCache = 8;  // items per thread kept in registers between the passes

struct QuantArgs {
    const float* u;
    uint8_t* ws;
    unsigned* zero;  // words cleared for the tcgen05 kernel's group counters (or null)
    int nzero;
    DecodePlan p;
};

__device__ __forceinline__ float4 load_item(const float* uc, int it) {
    const float* q = uc + 32 * (it >> 3) + (it & 7);
    return make_float4(q[0], q[8], q[16], q[24]);
}

__device__ __forceinline__ unsigned absbits(float x) { return __float_as_uint(x) & 0x7fffffffu; }

__device__ __forceinline__ unsigned absmax4(const float4& v) {
    return max(max(absbits(v.x), absbits(v.y)), max(absbits(v.z), absbits(v.w)));
}

// u_q of one element in the column's mode; sa * sb = 2^F in two exact factors.
__device__ __forceinline__ int quant1(float x, int mode, float sa, float sb) {
    if (mode == kColFinite) return __float2int_rn((x * sa) * sb);
    if (mode == kColInf) return isinf(x) ? (x > 0.f ? 1 : -1) : 0;
    return 0;
}

__global__ void __launch_bounds__(kQThreads, 1) quant_kernel(const QuantArgs a) {
    // u is written by the kernel before this one; the workspace may still be read
    // by the previous call's contraction. Wait for both, then let the contraction
    // launch (its early reads of the weights therefore also follow the kernel
    // before this call).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const DecodePlan& p = a.p;
    extern __shared__ StepSum s_steps[];  // p.nsteps
    __shared__ unsigned s_max;
    const int c = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const float* uc = a.u + (size_t)c * p.K;
    const int nitems = p.kw * 8;

    if (tid == 0) s_max = 0u;
    for (int i = tid; i < p.nsteps; i += kQThreads) {
        s_steps[i].S = 0;
        s_steps[i].ninf = 0;
        s_steps[i].pad = 0;
    }
    if (c == 0)
        for (int i = tid; i < a.nzero; i += kQThreads) a.zero[i] = 0u;
    __syncthreads();

    // ---- pass 1: the largest |u| as float bits (NaN > Inf > any finite value)
    float4 v[kQCache];
    unsigned mx = 0u;
#pragma unroll
    for (int r = 0; r < kQCache; ++r) {
        const int it = r * kQThreads + tid;
        v[r] = it < nitems ? load_item(uc, it) : make_float4(0.f, 0.f, 0.f, 0.f);
        mx = max(mx, absmax4(v[r]));
    }
    for (int it = kQCache * kQThreads + tid; it < nitems; it += kQThreads) mx = max(mx, absmax4(load_item(uc, it)));
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) atomicMax(&s_max, mx);
    __syncthreads();

    const unsigned cmax = s_max;
    const int mode = cmax > 0x7f800000u ? kColNaN : cmax == 0x7f800000u ? kColInf : kColFinite;
    // cmax < 2^e (zero and subnormal maxima: e = -126); F = 30 - e keeps |u_q| <= 2^30
    const int E = (int)(cmax >> 23);
    const int F = mode == kColFinite ? 30 - (E == 0 ? -126 : E - 126) : 0;
    const int Fa = F > 127 ? F / 2 : F;  // 2^F as two float factors when it exceeds the float range
    const float sa = __int_as_float((127 + Fa) << 23), sb = __int_as_float((127 + F - Fa) << 23);

    // ---- pass 2: digits, step sums, Inf counts
    auto convert = [&](int it, const float4& x) {
        const int q0 = quant1(x.x, mode, sa, sb), q1 = quant1(x.y, mode, sa, sb);
        const int q2 = quant1(x.z, mode, sa, sb), q3 = quant1(x.w, mode, sa, sb);
        const bool live = it < nitems;
        // balanced digits: byte pl of t is digit pl
        const uint32_t t0 = ((uint32_t)q0 + 0x80808080u) ^ 0x80808080u;
        const uint32_t t1 = ((uint32_t)q1 + 0x80808080u) ^ 0x80808080u;
        const uint32_t t2 = ((uint32_t)q2 + 0x80808080u) ^ 0x80808080u;
        const uint32_t t3 = ((uint32_t)q3 + 0x80808080u) ^ 0x80808080u;
        const uint32_t a01 = __byte_perm(t0, t1, 0x5140), a23 = __byte_perm(t2, t3, 0x5140);  // bytes 0, 1
        const uint32_t b01 = __byte_perm(t0, t1, 0x7362), b23 = __byte_perm(t2, t3, 0x7362);  // bytes 2, 3
        const uint32_t P[kPlanes] = {__byte_perm(a01, a23, 0x5410), __byte_perm(a01, a23, 0x7632),
                                     __byte_perm(b01, b23, 0x5410), __byte_perm(b01, b23, 0x7632)};
        if (live) {
            const int x = it >> 3, j = it & 7;
#pragma unroll
            for (int pl = 0; pl < kPlanes; ++pl) {
                *reinterpret_cast<uint32_t*>(a.ws + p.off_planes + mma_digit_offset(p, c, pl, x, j)) = P[pl];
            }
        }
        // |q0 + .. + q3| <= 2^32: reduced as 16-bit low parts and the high rest
        const long long qs = (long long)q0 + q1 + q2 + q3;
        const unsigned lo = __reduce_add_sync(0xffffffffu, (unsigned)(qs & 0xffff));
        const int hi = __reduce_add_sync(0xffffffffu, (int)(qs >> 16));
        const int ni = __reduce_add_sync(0xffffffffu, live ? (int)isinf(x.x) + (int)isinf(x.y) + (int)isinf(x.z) +
                                                                  (int)isinf(x.w)
                                                            : 0);
        // a warp's items are four words of one step (or past the end, all zero)
        const int step = (it - lane) >> 7;
        if (lane == 0 && step < p.nsteps) {
            atomicAdd(reinterpret_cast<unsigned long long*>(&s_steps[step].S),
                      (unsigned long long)(((long long)hi << 16) + (long long)lo));
            if (ni) atomicAdd(&s_steps[step].ninf, ni);
        }
    };
#pragma unroll
    for (int r = 0; r < kQCache; ++r) {
        const int it = r * kQThreads + tid;
        if (it - lane < nitems) convert(it, v[r]);  // warp-uniform
    }
    for (int it = kQCache * kQThreads + tid; it - lane < nitems; it += kQThreads)
        convert(it, it < nitems ? load_item(uc, it) : make_float4(0.f, 0.f, 0.f, 0.f));
    __syncthreads();

    StepSum* steps = reinterpret_cast<StepSum*>(a.ws + p.off_steps) + (size_t)c * p.nsteps;
    for (int i = tid; i < p.nsteps; i += kQThreads) steps[i] = s_steps[i];
    if (tid == 0) {
        ColHeader h;
        h.F = F;
        h.mode = mode;
        h.pad0 = h.pad1 = 0;
        reinterpret_cast<ColHeader*>(a.ws + p.off_hdr)[c] = h;
    }
}


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

namespace {
}  // namespace

cudaError_t launch_quant(const float* u, const DecodePlan& p, void* ws, unsigned* zero, int nzero, cudaStream_t st) {
    const size_t smem = (size_t)p.nsteps * sizeof(StepSum);
    static size_t granted[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (smem > 48 * 1024 && (dev >= 64 || granted[dev] < smem)) {
        cudaError_t e = cudaFuncSetAttribute(quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) granted[dev] = smem;
    }
    QuantArgs a;
    a.u = u;
    a.ws = static_cast<uint8_t*>(ws);
    a.zero = zero;
    a.nzero = nzero;
    a.p = p;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.batch, 1, 1);
    cfg.blockDim = dim3(kQThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, quant_kernel, a);
}

}  // namespace lq
