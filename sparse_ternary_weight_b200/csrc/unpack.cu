// unpack.cu -- packed planes -> dense bf16 W[n][k] = RNE(t[n][k] * alpha).
//
// The inverse of the 32-state block code ("Sherry: Hardware-Efficient 1.25-Bit
// Ternary Quantization via Fine-grained Sparsification", digest paragraph on the
// 5-bit packing: zero position x signs of the other two relative to the first
// nonzero, plus one global sign bit) times the scale of the weight's domain.
// HBM-bound on the 2 B/weight write; one thread expands one 32-weight word.
#include "common.cuh"

#include <cuda_bf16.h>

namespace sherry {

// 4 bf16 of one block -> two packed 32-bit halves
__device__ __forceinline__ uint2 expand_block(uint32_t nib, uint32_t g, uint32_t pos, uint32_t neg) {
    const uint32_t z = nib >> 2;
    const uint32_t d1 = (nib >> 1) & 1u, d2 = nib & 1u;
    // negative bits of the kept weights in position order, then reinsert the zero slot
    const uint32_t k3 = g | ((g ^ d1) << 1) | ((g ^ d2) << 2);
    const uint32_t negs = (k3 & ((1u << z) - 1u)) | ((k3 >> z) << (z + 1));
    uint32_t h[4];
#pragma unroll
    for (uint32_t i = 0; i < 4; ++i) h[i] = (i == z) ? 0u : (((negs >> i) & 1u) ? neg : pos);
    return make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
}

__global__ void __launch_bounds__(256)
k_unpack(const uint32_t* __restrict__ idx, const uint8_t* __restrict__ sgn, const float* __restrict__ scales,
         int64_t N, int K, int granularity, int group, uint16_t* __restrict__ out) {
    const int words = K >> 5;
    const int64_t total = N * (int64_t)words;
    for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
         w += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = w / words;
        const int wi = (int)(w - n * words);
        int64_t si;
        if (granularity == SHERRY_PER_TENSOR)
            si = 0;
        else if (granularity == SHERRY_PER_CHANNEL)
            si = n;
        else
            si = n * (K / group) + (int64_t)wi * 32 / group;
        const float a = __ldg(scales + si);
        const uint32_t pos = __bfloat16_as_ushort(__float2bfloat16_rn(a));
        const uint32_t neg = pos ^ 0x8000u;  // RNE is symmetric in the sign
        const uint32_t code = __ldg(idx + w);
        const uint32_t sb = __ldg(sgn + w);
        uint4 o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint2 lo = expand_block((code >> (8 * q)) & 15u, (sb >> (2 * q)) & 1u, pos, neg);
            const uint2 hi = expand_block((code >> (8 * q + 4)) & 15u, (sb >> (2 * q + 1)) & 1u, pos, neg);
            o[q] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
        uint4* dst = reinterpret_cast<uint4*>(out + w * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) __stcs(dst + q, o[q]);
    }
}

int unpack_launch(const uint32_t* idx, const uint8_t* sgn, const float* scales, int64_t N, int64_t K,
                  int granularity, int group, uint16_t* out, cudaStream_t stream, int num_sms) {
    const int64_t total = N * (K / 32);
    if (total == 0) return SHERRY_OK;
    int64_t blocks = (total + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    k_unpack<<<(unsigned)blocks, 256, 0, stream>>>(idx, sgn, scales, N, (int)K, granularity, group, out);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

}  // namespace sherry
