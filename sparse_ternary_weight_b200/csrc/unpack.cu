// unpack.cu -- packed planes -> dense bf16 W[n][k] = RNE(t[n][k] * alpha), or
// fp32 t[n][k] * alpha (the quantiser's forward output for per-tensor scales).
//
// The inverse of the 32-state block code ("Sherry: Hardware-Efficient 1.25-Bit
// Ternary Quantization via Fine-grained Sparsification", digest paragraph on the
// 5-bit packing: zero position x signs of the other two relative to the first
// nonzero, plus one global sign bit) times the scale of the weight's domain.
// HBM-bound on the 2 B/weight write: each warp writes 512 contiguous bytes, one
// selector-table lookup and two byte permutes per block of 4 weights.
#include "common.cuh"

#include <cuda_bf16.h>

#include <mutex>

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

constexpr int kUSeg = 4;  // 8-word segments per warp and pass

struct UProb {
    const uint32_t* idx;
    const uint8_t* sgn;
    const float* scales;
    void* out;            // bf16 [N][K], or fp32 [N][K] when f32
    int f32;
    int64_t words_total;  // N * K / 32
    int64_t seg_begin;    // first 8-word segment of this problem in the launch
    int words, granularity, gwords;
};

template <int MAXP>
struct UParams {
    int count;
    int64_t total_segs;
    UProb p[MAXP];
};

// One warp writes 512 contiguous output bytes (8 packed words of one problem);
// lane l expands blocks 2(l % 4) and 2(l % 4) + 1 of word 8 s + l / 4 into 16 bytes.
// Segments of all problems of the launch are dealt to the warps round-robin.
template <int MAXP>
__global__ void __launch_bounds__(256) k_unpack(const __grid_constant__ UParams<MAXP> P) {
    __shared__ uint32_t sel[32];
    __shared__ float4 tpat[32];  // ternary values of each block code (fp32 output)
    if (threadIdx.x < 32) {
        const uint32_t s4 = block_selector(threadIdx.x & 15u, threadIdx.x >> 4);
        sel[threadIdx.x] = s4;
        // the selector's (lo, hi) picks: (3, 3) = 0, (0, 1) = +1, (0, 2) = -1
        float t[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t hi = (s4 >> (8 * i + 4)) & 0xfu;
            t[i] = hi == 3u ? 0.0f : (hi == 2u ? -1.0f : 1.0f);
        }
        tpat[threadIdx.x] = make_float4(t[0], t[1], t[2], t[3]);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int q = lane & 3;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    int pi = 0;  // problem cursor: segments are visited in increasing order
    // kUSeg consecutive segments per warp and pass: all their loads are issued before
    // any expansion, so several DRAM reads per warp are in flight at once
    for (int64_t sg = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); sg * kUSeg < P.total_segs;
         sg += nwarps) {
        uint32_t code[kUSeg], sbits[kUSeg], R[kUSeg];
        int64_t off[kUSeg];  // output element of the lane's 8 weights, or -1
        const UProb* pp[kUSeg];
#pragma unroll
        for (int j = 0; j < kUSeg; ++j) {
            const int64_t seg = sg * kUSeg + j;
            off[j] = -1;
            code[j] = sbits[j] = R[j] = 0u;
            pp[j] = &P.p[0];
            if (seg < P.total_segs) {
                while (pi + 1 < P.count && P.p[pi + 1].seg_begin <= seg) ++pi;
                const UProb& pr = P.p[pi];
                const int64_t w = (seg - pr.seg_begin) * 8 + (lane >> 2);
                if (w < pr.words_total) {
                    const bool small = pr.words_total <= 0xffffffffLL;
                    int64_t si;
                    if (pr.granularity == SHERRY_PER_TENSOR)
                        si = 0;
                    else if (pr.granularity == SHERRY_PER_CHANNEL)
                        si = small ? (int64_t)((uint32_t)w / (uint32_t)pr.words) : w / pr.words;
                    else
                        si = small ? (int64_t)((uint32_t)w / (uint32_t)pr.gwords) : w / pr.gwords;  // (32 w) / group
                    code[j] = __ldg(pr.idx + w);
                    sbits[j] = __ldg(pr.sgn + w);
                    R[j] = __float_as_uint(__ldg(pr.scales + si));
                    off[j] = w * 32 + q * 8;
                    pp[j] = &pr;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kUSeg; ++j) {
            if (off[j] >= 0 && pp[j]->f32) {
                const float a = __uint_as_float(R[j]);
                const uint32_t byte = (code[j] >> (8 * q)) & 0xffu;
                const uint32_t sb = sbits[j] >> (2 * q);
                const float4 t0 = tpat[(byte & 15u) | ((sb & 1u) << 4)];
                const float4 t1 = tpat[(byte >> 4) | ((sb & 2u) << 3)];
                float4* o = reinterpret_cast<float4*>(static_cast<float*>(pp[j]->out) + off[j]);
                __stcs(o, make_float4(t0.x * a, t0.y * a, t0.z * a, t0.w * a));
                __stcs(o + 1, make_float4(t1.x * a, t1.y * a, t1.z * a, t1.w * a));
            } else if (off[j] >= 0) {
                const uint32_t pos = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(R[j])));
                const uint32_t r4 = pos | (((pos >> 8) | 0x80u) << 16);  // RNE is symmetric in the sign
                const uint32_t byte = (code[j] >> (8 * q)) & 0xffu;
                const uint32_t sb = sbits[j] >> (2 * q);
                const uint32_t s0 = sel[(byte & 15u) | ((sb & 1u) << 4)];
                const uint32_t s1 = sel[(byte >> 4) | ((sb & 2u) << 3)];
                uint4 o;
                o.x = __byte_perm(r4, r4, s0 & 0xffffu);
                o.y = __byte_perm(r4, r4, s0 >> 16);
                o.z = __byte_perm(r4, r4, s1 & 0xffffu);
                o.w = __byte_perm(r4, r4, s1 >> 16);
                __stcs(reinterpret_cast<uint4*>(static_cast<uint16_t*>(pp[j]->out) + off[j]), o);
            }
        }
    }
}

template <int MAXP>
static int unpack_launch_t(const sherry_unpack_desc* d, const int* f32, int count, cudaStream_t stream,
                           int num_sms) {
    static UParams<MAXP> P;
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    int64_t segs = 0;
    int n = 0;
    for (int i = 0; i < count; ++i) {
        const int64_t total = d[i].N * (d[i].K / 32);
        if (total == 0) continue;
        UProb& p = P.p[n++];
        p.idx = d[i].idx;
        p.sgn = d[i].sgn;
        p.scales = d[i].scales;
        p.out = d[i].W_out;
        p.f32 = f32 ? f32[i] : 0;
        p.words_total = total;
        p.seg_begin = segs;
        p.words = (int)(d[i].K / 32);
        p.granularity = d[i].granularity;
        p.gwords = d[i].granularity == SHERRY_PER_GROUP ? d[i].group / 32 : 1;
        segs += (total + 7) / 8;
    }
    if (segs == 0) return SHERRY_OK;
    P.count = n;
    P.total_segs = segs;
    int64_t blocks = (segs + 8 * kUSeg - 1) / (8 * kUSeg);  // 8 warps per block, kUSeg segments each per pass
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    k_unpack<MAXP><<<(unsigned)blocks, 256, 0, stream>>>(P);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

int unpack_launch_ex(const sherry_unpack_desc* descs, const int* f32, int count, cudaStream_t stream, int num_sms) {
    if (count <= 1) return unpack_launch_t<1>(descs, f32, count, stream, num_sms);
    if (count <= 16) return unpack_launch_t<16>(descs, f32, count, stream, num_sms);
    return unpack_launch_t<SHERRY_MAX_BATCH>(descs, f32, count, stream, num_sms);
}

int unpack_launch(const sherry_unpack_desc* descs, int count, cudaStream_t stream, int num_sms) {
    return unpack_launch_ex(descs, nullptr, count, stream, num_sms);
}

}  // namespace sherry
