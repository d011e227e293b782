// Sign packing for the 1-bit matrix W_q (LiftQuant paper note, "Key designs" 1
// and 4: D one-bit signs per d weights). Layout: 32 signs per uint32, least
// significant bit first along the lifted axis, bit 1 = +1, rows [out][K/32].
//
// Both kernels are pure streaming: one thread per packed word, 32 int8 signs
// moved as two 16-byte vectors. Grids are sized in multiples of the SM count
// and grid-stride over the words.
#include "lq_debug.cuh"
#include "lq_internal.h"

namespace lq {
namespace {

// +1 (any positive int8) -> bit 1. The four bytes of x hold signs k..k+3.
__device__ __forceinline__ uint32_t positive_bytes_to_bits(uint32_t x) {
    // a byte b is positive iff b != 0 and its top bit is clear
    uint32_t nonzero = ((x & 0x7f7f7f7fu) + 0x7f7f7f7fu) | x;  // top bit set iff byte != 0
    uint32_t pos = nonzero & ~x & 0x80808080u;                 // top bit set iff byte > 0
    // gather the four top bits (positions 7, 15, 23, 31) into bits 0..3
    return ((pos >> 7) & 1u) | ((pos >> 14) & 2u) | ((pos >> 21) & 4u) | ((pos >> 28) & 8u);
}

__global__ void __launch_bounds__(256) pack_kernel(const int8_t* __restrict__ signs, long long nwords,
                                                   uint32_t* __restrict__ packed) {
    for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < nwords;
         w += (long long)gridDim.x * blockDim.x) {
        const uint4* src = reinterpret_cast<const uint4*>(signs + w * 32);
        uint4 lo = __ldg(src), hi = __ldg(src + 1);
        uint32_t v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) word |= positive_bytes_to_bits(v[i]) << (4 * i);
        if (LQ_IN_BOUNDS(w, nwords)) packed[w] = word;
    }
}

// bit -> 0x01 (+1) or 0xff (-1) for the four bits at positions 0..3 of n.
__device__ __forceinline__ uint32_t bits_to_pm1_bytes(uint32_t n) {
    uint32_t spread = (n & 1u) | ((n & 2u) << 7) | ((n & 4u) << 14) | ((n & 8u) << 21);  // 0x01 per set bit
    // set bit -> 0x01, clear bit -> 0xff
    return spread | ((spread ^ 0x01010101u) * 0xffu);
}

__global__ void __launch_bounds__(256) unpack_kernel(const uint32_t* __restrict__ packed, long long nwords,
                                                     int8_t* __restrict__ signs) {
    for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < nwords;
         w += (long long)gridDim.x * blockDim.x) {
        uint32_t word = __ldg(packed + w);
        uint32_t v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = bits_to_pm1_bytes((word >> (4 * i)) & 0xfu);
        if (!LQ_IN_BOUNDS(w * 32 + 31, nwords * 32)) continue;
        uint4* dst = reinterpret_cast<uint4*>(signs + w * 32);
        dst[0] = make_uint4(v[0], v[1], v[2], v[3]);
        dst[1] = make_uint4(v[4], v[5], v[6], v[7]);
    }
}

int grid_for(long long n, int threads) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long want = (n + threads - 1) / threads;
    long long cap = (long long)sms * 8;
    return (int)(want < cap ? (want < 1 ? 1 : want) : cap);
}

}  // namespace

cudaError_t launch_pack(const int8_t* signs, int out, int K, uint32_t* packed, cudaStream_t st) {
    long long nwords = (long long)out * (K / 32);
    pack_kernel<<<grid_for(nwords, 256), 256, 0, st>>>(signs, nwords, packed);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const uint32_t* packed, int out, int K, int8_t* signs, cudaStream_t st) {
    long long nwords = (long long)out * (K / 32);
    unpack_kernel<<<grid_for(nwords, 256), 256, 0, st>>>(packed, nwords, signs);
    return cudaGetLastError();
}

}  // namespace lq

LQ_DEBUG_FLAG_TAKE(debug_take_pack)
