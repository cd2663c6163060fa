// unpack.cu -- packed planes -> dense bf16 W[n][k] = RNE(t[n][k] * alpha).
//
// The inverse of the 32-state block code ("Sherry: Hardware-Efficient 1.25-Bit
// Ternary Quantization via Fine-grained Sparsification", digest paragraph on the
// 5-bit packing: zero position x signs of the other two relative to the first
// nonzero, plus one global sign bit) times the scale of the weight's domain.
// HBM-bound on the 2 B/weight write: each warp writes 512 contiguous bytes, one
// selector-table lookup and two byte permutes per block of 4 weights.
#include "common.cuh"

#include <cuda_bf16.h>

namespace sherry {

// Byte-permute selectors of one block code (nibble + 16 G): the block's 4 bf16
// outputs are bytes of R = {lo(a), hi(a), hi(a) | 0x80, 0} with a = bf16(alpha):
// +alpha = bytes (0, 1), -alpha = (0, 2), 0 = (3, 3).  Low 16 bits: weights 0, 1;
// high 16 bits: weights 2, 3.
__device__ __forceinline__ uint32_t block_selector(uint32_t nib, uint32_t g) {
    const uint32_t z = nib >> 2;
    const uint32_t d1 = (nib >> 1) & 1u, d2 = nib & 1u;
    // negative flags of the kept weights in position order, then the zero slot reinserted
    const uint32_t k3 = g | ((g ^ d1) << 1) | ((g ^ d2) << 2);
    const uint32_t negs = (k3 & ((1u << z) - 1u)) | ((k3 >> z) << (z + 1));
    uint32_t sel = 0;
#pragma unroll
    for (uint32_t i = 0; i < 4; ++i) {
        const uint32_t pair = (i == z) ? 0x33u : (((negs >> i) & 1u) ? 0x20u : 0x10u);  // (lo, hi) byte picks
        sel |= pair << (8 * i);
    }
    return sel;
}

// One warp writes 512 contiguous output bytes (8 packed words); lane l expands
// blocks 2(l % 4) and 2(l % 4) + 1 of word 8 s + l / 4 into 16 bytes.
__global__ void __launch_bounds__(256)
k_unpack(const uint32_t* __restrict__ idx, const uint8_t* __restrict__ sgn, const float* __restrict__ scales,
         int64_t total_words, int words, int granularity, int gwords, uint16_t* __restrict__ out) {
    __shared__ uint32_t sel[32];
    if (threadIdx.x < 32) sel[threadIdx.x] = block_selector(threadIdx.x & 15u, threadIdx.x >> 4);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int q = lane & 3;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const bool small = total_words <= 0xffffffffLL;
    for (int64_t seg = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); seg * 8 < total_words;
         seg += nwarps) {
        const int64_t w = seg * 8 + (lane >> 2);
        if (w >= total_words) continue;
        int64_t si;
        if (granularity == SHERRY_PER_TENSOR)
            si = 0;
        else if (granularity == SHERRY_PER_CHANNEL)
            si = small ? (int64_t)((uint32_t)w / (uint32_t)words) : w / words;
        else
            si = small ? (int64_t)((uint32_t)w / (uint32_t)gwords) : w / gwords;  // (32 w) / group
        const uint32_t pos = __bfloat16_as_ushort(__float2bfloat16_rn(__ldg(scales + si)));
        const uint32_t R = pos | (((pos >> 8) | 0x80u) << 16);  // RNE is symmetric in the sign
        const uint32_t byte = (__ldg(idx + w) >> (8 * q)) & 0xffu;
        const uint32_t sb = (uint32_t)__ldg(sgn + w) >> (2 * q);
        const uint32_t s0 = sel[(byte & 15u) | ((sb & 1u) << 4)];
        const uint32_t s1 = sel[(byte >> 4) | ((sb & 2u) << 3)];
        uint4 o;
        o.x = __byte_perm(R, R, s0 & 0xffffu);
        o.y = __byte_perm(R, R, s0 >> 16);
        o.z = __byte_perm(R, R, s1 & 0xffffu);
        o.w = __byte_perm(R, R, s1 >> 16);
        __stcs(reinterpret_cast<uint4*>(out + w * 32 + q * 8), o);
    }
}

int unpack_launch(const uint32_t* idx, const uint8_t* sgn, const float* scales, int64_t N, int64_t K,
                  int granularity, int group, uint16_t* out, cudaStream_t stream, int num_sms) {
    const int64_t total = N * (K / 32);
    if (total == 0) return SHERRY_OK;
    int64_t blocks = (total + 63) / 64;  // 8 warps x 8 words
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    const int gwords = granularity == SHERRY_PER_GROUP ? group / 32 : 1;
    k_unpack<<<(unsigned)blocks, 256, 0, stream>>>(idx, sgn, scales, total, (int)(K / 32), granularity, gwords,
                                                   out);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

}  // namespace sherry
