// quantize.cu -- greedy Sparse-AbsMean quantise + 5-bit pack (3:4 sparsity).
//
// "Sherry: Hardware-Efficient 1.25-Bit Ternary Quantization via Fine-grained
// Sparsification" (digest paragraph on the 3:4 rule): in each block of 4 the
// smallest |w| is zeroed, the other three keep their signs, and the scale is
// the mean |w| of the kept weights; a block is 1 sign bit + 4 lookup bits.
// "Sherry, Tequila and Fairies in Python", section 1.1: the scale domain is a
// group of `group` weights along K, a row, or the whole tensor, and the
// denominator is max(L * 3/4, 1) for a domain of L weights.
//
// Kernel 1 (one CTA per row, HBM-bound on the read of W): each lane owns four
// blocks of 4 (16 consecutive weights, half a packed word), finds each zero
// position and the negative-sign bits in registers and takes the 5-bit code
// (nibble + 16 G) from a 64-entry table indexed by (zero position, sign bits);
// one xor shuffle with the partner lane completes the word's nibbles, its sign
// byte and its masked |w| sum (the lower five levels of the canonical pairwise
// tree, in that order).  Word sums sit in shared memory; the scales are then
// the upper levels of the tree over each domain.
// Kernel 2 (per-tensor only): one CTA folds the per-row subtree sums.
#include "common.cuh"

namespace sherry {

constexpr int kQThreads = 256;
constexpr int kQUnroll = 2;  // warp-steps (16 weights per lane each) in flight

// 5-bit code (nibble 4z + 2 d1 + d2, plus 16 G) of a block whose smallest |w|
// is at z and whose negative weights are the set bits of `neg` (w < 0; -0.0 is
// not negative): the kept signs in position order are k0 k1 k2, G = k0,
// d1 = k1 ^ k0, d2 = k2 ^ k0.
__device__ __forceinline__ uint32_t code_of(uint32_t z, uint32_t neg) {
    const uint32_t low = neg & ((1u << z) - 1u);
    const uint32_t k3 = low | ((neg >> (z + 1)) << z);
    const uint32_t g = k3 & 1u;
    const uint32_t d1 = ((k3 >> 1) ^ k3) & 1u;
    const uint32_t d2 = ((k3 >> 2) ^ k3) & 1u;
    return 4u * z + 2u * d1 + d2 + 16u * g;
}

// one block of 4: code from the table, masked magnitude sum (m0 + m1) + (m2 + m3)
__device__ __forceinline__ uint32_t encode4(float w0, float w1, float w2, float w3, const uint8_t* ctab,
                                            float& mag) {
    const float a0 = fabsf(w0), a1 = fabsf(w1), a2 = fabsf(w2), a3 = fabsf(w3);
    // first index of the minimum |w| (strict < keeps the earlier index on ties)
    uint32_t z = 0;
    float m = a0;
    if (a1 < m) { z = 1; m = a1; }
    if (a2 < m) { z = 2; m = a2; }
    if (a3 < m) { z = 3; }
    const uint32_t neg = (w0 < 0.0f ? 1u : 0u) | (w1 < 0.0f ? 2u : 0u) | (w2 < 0.0f ? 4u : 0u) |
                         (w3 < 0.0f ? 8u : 0u);
    mag = ((z == 0 ? 0.0f : a0) + (z == 1 ? 0.0f : a1)) + ((z == 2 ? 0.0f : a2) + (z == 3 ? 0.0f : a3));
    return ctab[(z << 4) | neg];
}

// 16 consecutive weights (4 blocks) per lane
template <bool kBF16>
struct WLoad;

template <>
struct WLoad<false> {
    struct T { float4 q[4]; };
    __device__ __forceinline__ static T load(const void* W, int64_t off16) {
        const float4* p = reinterpret_cast<const float4*>(W) + off16 * 4;
        T v;
#pragma unroll
        for (int i = 0; i < 4; ++i) v.q[i] = __ldcs(p + i);
        return v;
    }
    __device__ __forceinline__ static void block(const T& v, int j, float& a, float& b, float& c, float& d) {
        a = v.q[j].x; b = v.q[j].y; c = v.q[j].z; d = v.q[j].w;
    }
    __device__ __forceinline__ static T zero() {
        T v;
#pragma unroll
        for (int i = 0; i < 4; ++i) v.q[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        return v;
    }
};

template <>
struct WLoad<true> {
    struct T { uint4 q[2]; };
    __device__ __forceinline__ static T load(const void* W, int64_t off16) {
        const uint4* p = reinterpret_cast<const uint4*>(W) + off16 * 2;
        T v;
        v.q[0] = __ldcs(p);
        v.q[1] = __ldcs(p + 1);
        return v;
    }
    __device__ __forceinline__ static void block(const T& v, int j, float& a, float& b, float& c, float& d) {
        const uint4& u = v.q[j >> 1];
        const uint32_t x = (j & 1) ? u.z : u.x, y = (j & 1) ? u.w : u.y;
        a = __uint_as_float(x << 16);
        b = __uint_as_float(x & 0xffff0000u);
        c = __uint_as_float(y << 16);
        d = __uint_as_float(y & 0xffff0000u);
    }
    __device__ __forceinline__ static T zero() {
        T v;
        v.q[0] = v.q[1] = make_uint4(0u, 0u, 0u, 0u);
        return v;
    }
};

// granularity of the scale written by kernel 1
enum QMode { kQGroup = 0, kQChannel = 1, kQTensorPartials = 2 };

template <bool kBF16, int kMode>
__global__ void __launch_bounds__(kQThreads)
k_quantize_rows(const void* __restrict__ W, int K, uint32_t* __restrict__ idx,
                uint8_t* __restrict__ sgn, float* __restrict__ out,
                int gw /* group words (per-group) or chunk words (per-tensor) */, float D) {
    extern __shared__ float wsum[];  // K/32 word sums of masked |w|
    __shared__ uint8_t ctab[64];     // 5-bit code by (zero position, negative bits)
    using L = WLoad<kBF16>;
    const int64_t n = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int words = K >> 5;
    const int n16 = K >> 4;                  // 16-weight pieces (two per word)
    const int nsteps = (n16 + 31) >> 5;      // 512 weights = 16 words = one warp-step
    const int64_t row16 = n * (int64_t)n16;
    const int64_t row_word = n * (int64_t)words;
    if (threadIdx.x < 64) ctab[threadIdx.x] = (uint8_t)code_of(threadIdx.x >> 4, threadIdx.x & 15u);
    __syncthreads();

    for (int c0 = warp; c0 < nsteps; c0 += 8 * kQUnroll) {
        typename L::T v[kQUnroll];
#pragma unroll
        for (int u = 0; u < kQUnroll; ++u) {
            const int piece = (c0 + 8 * u) * 32 + lane;
            v[u] = (c0 + 8 * u < nsteps && piece < n16) ? L::load(W, row16 + piece) : L::zero();
        }
#pragma unroll
        for (int u = 0; u < kQUnroll; ++u) {
            const int c = c0 + 8 * u;
            if (c >= nsteps) continue;  // warp-uniform
            const int piece = c * 32 + lane;
            const int half = lane & 1;
            uint32_t nib = 0, sg = 0;
            float m4[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float w0, w1, w2, w3;
                L::block(v[u], j, w0, w1, w2, w3);
                const uint32_t code = encode4(w0, w1, w2, w3, ctab, m4[j]);
                nib |= (code & 15u) << (4 * j);
                sg |= (code >> 4) << j;
            }
            // half 0 holds blocks 0..3 of the word, half 1 blocks 4..7
            uint32_t word = nib << (16 * half);
            word |= __shfl_xor_sync(kFull, word, 1);
            uint32_t sb = sg << (4 * half);
            sb |= __shfl_xor_sync(kFull, sb, 1);
            float s = (m4[0] + m4[1]) + (m4[2] + m4[3]);
            const float o = __shfl_xor_sync(kFull, s, 1);
            s = half ? o + s : s + o;  // ((b0 + b1) + (b2 + b3)) + ((b4 + b5) + (b6 + b7))
            // both lanes of a word are valid or neither (K % 32 == 0)
            if (half == 0 && piece < n16) {
                const int w = piece >> 1;
                idx[row_word + w] = word;
                sgn[row_word + w] = (uint8_t)sb;
                wsum[w] = s;
            }
        }
    }
    __syncthreads();

    if (kMode == kQGroup) {
        // one scale per group of gw words: upper tree levels over the word sums
        const int ngroups = words / gw;
        for (int j = threadIdx.x; j < ngroups; j += kQThreads) {
            float S;
            const float* v = wsum + j * gw;
            if (gw == 4) {
                S = (v[0] + v[1]) + (v[2] + v[3]);
            } else if (gw == 1) {
                S = v[0];
            } else if (gw == 2) {
                S = v[0] + v[1];
            } else {
                S = tree_sum_seq(v, gw);
            }
            out[n * ngroups + j] = S / D;
        }
    } else if (kMode == kQChannel) {
        if (warp == 0) {
            float S = warp_tree_sum(wsum, words);
            if (lane == 0) out[n] = S / D;
        }
    } else {
        // per-tensor: sums of the aligned 2^j-weight subtrees that tile the row
        const int nparts = words / gw;
        for (int j = warp; j < nparts; j += kQThreads / 32) {
            float S = warp_tree_sum(wsum + j * gw, gw);
            if (lane == 0) out[n * nparts + j] = S;
        }
    }
}

// Per-tensor finalize: canonical tree over `count` subtree sums, then / D.
__global__ void __launch_bounds__(1024)
k_tensor_scale(const float* __restrict__ parts, int64_t count, float D, float* __restrict__ scale) {
    __shared__ float red[32];
    const int t = threadIdx.x;
    const int64_t P = pow2_ceil64(count > 0 ? count : 1);
    const int64_t seg = P > 1024 ? P / 1024 : 1;
    const int64_t lo = (int64_t)t * seg;
    float x = 0.0f;
    if (lo < count) {
        int64_t cnt = count - lo;
        if (cnt > seg) cnt = seg;
        // sequential canonical tree over an aligned segment (seg is a power of two)
        float st[40];
        int lv[40];
        int top = 0;
        for (int64_t i = 0; i < cnt; ++i) {
            float y = __ldcg(parts + lo + i);
            int l = 0;
            while (top > 0 && lv[top - 1] == l) {
                y = st[top - 1] + y;
                --top;
                ++l;
            }
            st[top] = y;
            lv[top] = l;
            ++top;
        }
        x = st[top - 1];
        for (int q = top - 2; q >= 0; --q) x = st[q] + x;
    }
    for (int off = 1; off < 32; off <<= 1) x = x + __shfl_xor_sync(kFull, x, off);
    if ((t & 31) == 0) red[t >> 5] = x;
    __syncthreads();
    if (t < 32) {
        float y = red[t];
        for (int off = 1; off < 32; off <<= 1) y = y + __shfl_xor_sync(kFull, y, off);
        if (t == 0) *scale = y / D;
    }
}

// ---- host side ---------------------------------------------------------------

// largest power of two dividing K, i.e. the subtree size that tiles both each
// row and the flattened tensor
static int64_t tensor_chunk(int64_t K) { return K & (-K); }

size_t quantize_workspace_bytes(int64_t N, int64_t K, int granularity) {
    if (granularity != SHERRY_PER_TENSOR) return 0;
    return (size_t)(N * (K / tensor_chunk(K))) * sizeof(float);
}

static float denom(int64_t L) {
    double d = (double)L / 4.0 * 3.0;
    if (d < 1.0) d = 1.0;
    return (float)d;
}

int quantize_pack_launch(const void* W, int w_dtype, int64_t N, int64_t K, int granularity, int group,
                         uint32_t* idx, uint8_t* sgn, float* scales, void* workspace,
                         cudaStream_t stream) {
    const size_t smem = (size_t)(K / 32) * sizeof(float);
    const bool bf = (w_dtype == SHERRY_BF16);
    if (granularity == SHERRY_PER_GROUP) {
        if (N == 0) return SHERRY_OK;
        const int gw = group / 32;
        if (bf)
            k_quantize_rows<true, kQGroup><<<(unsigned)N, kQThreads, smem, stream>>>(
                W, (int)K, idx, sgn, scales, gw, denom(group));
        else
            k_quantize_rows<false, kQGroup><<<(unsigned)N, kQThreads, smem, stream>>>(
                W, (int)K, idx, sgn, scales, gw, denom(group));
        SHERRY_LAUNCH_CHECK();
    } else if (granularity == SHERRY_PER_CHANNEL) {
        if (N == 0) return SHERRY_OK;
        if (bf)
            k_quantize_rows<true, kQChannel><<<(unsigned)N, kQThreads, smem, stream>>>(
                W, (int)K, idx, sgn, scales, 0, denom(K));
        else
            k_quantize_rows<false, kQChannel><<<(unsigned)N, kQThreads, smem, stream>>>(
                W, (int)K, idx, sgn, scales, 0, denom(K));
        SHERRY_LAUNCH_CHECK();
    } else {
        const int64_t c = tensor_chunk(K);
        float* parts = static_cast<float*>(workspace);
        if (N > 0) {
            if (bf)
                k_quantize_rows<true, kQTensorPartials><<<(unsigned)N, kQThreads, smem, stream>>>(
                    W, (int)K, idx, sgn, parts, (int)(c / 32), 0.0f);
            else
                k_quantize_rows<false, kQTensorPartials><<<(unsigned)N, kQThreads, smem, stream>>>(
                    W, (int)K, idx, sgn, parts, (int)(c / 32), 0.0f);
            SHERRY_LAUNCH_CHECK();
        }
        k_tensor_scale<<<1, 1024, 0, stream>>>(parts, N * (K / c), denom(N * K), scales);
        SHERRY_LAUNCH_CHECK();
    }
    return SHERRY_OK;
}

}  // namespace sherry
