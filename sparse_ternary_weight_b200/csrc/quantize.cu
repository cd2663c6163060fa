// quantize.cu -- greedy Sparse-AbsMean quantise + 5-bit pack (3:4 sparsity),
// and the quantiser's forward output (fake quantisation) in the same pass.
//
// "Sherry: Hardware-Efficient 1.25-Bit Ternary Quantization via Fine-grained
// Sparsification" (digest paragraph on the 3:4 rule): in each block of 4 the
// smallest |w| is zeroed, the other three keep their signs, and the scale is
// the mean |w| of the kept weights; a block is 1 sign bit + 4 lookup bits.
// "Sherry, Tequila and Fairies in Python", section 1.1: the scale domain is a
// group of `group` weights along K, a row, or the whole tensor, the
// denominator is max(L * 3/4, 1) for a domain of L weights, and the forward
// output (SherryNMQuant.forward) is sign * mask * scale.
//
// Kernel 1 (HBM-bound on the read of W): one launch for any number of weights
// of any element type and granularity; each CTA takes rows of the launch in
// turn (grid-stride).  Per row, each lane owns four blocks of 4 (16 consecutive
// weights, half a packed word), finds each zero position and the negative-sign
// bits in registers and takes the 5-bit code (nibble + 16 G) from a 64-entry
// table indexed by (zero position, sign bits); one xor shuffle with the
// partner lane completes the word's nibbles, its sign byte and its masked |w|
// sum (the lower five levels of the canonical pairwise tree, in that order).
// Word sums sit in shared memory; the scales are the upper levels of the tree
// over each domain.  With group or row scales the row's fake-quantised weights
// t * alpha (fp32 or bf16) are then written from the row's packed words, so W
// is read once.
// Kernel 2 (per-tensor only, one CTA per weight): folds the per-row subtree
// sums of a tensor into its scale.
#include "common.cuh"

#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <vector>

namespace sherry {

constexpr int kQThreads = 64;
constexpr int kQUnroll = 2;      // warp-steps (16 weights per lane each) in flight
constexpr int kQCtasPerSm = 28;  // CTAs per SM in the grid (two warps each: many rows in flight per SM)

// 5-bit code (nibble 4z + 2 d1 + d2, plus 16 G) of a block whose smallest |w|
// is at z and whose negative weights are the set bits of `neg` (w < 0; -0.0 is
// not negative): the kept signs in position order are k0 k1 k2, G = k0,
// d1 = k1 ^ k0, d2 = k2 ^ k0.
__host__ __device__ __forceinline__ uint32_t code_of(uint32_t z, uint32_t neg) {
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
    // first index of the minimum |w|, as a tournament of pairs (strict < keeps the
    // earlier index on ties, inside a pair and between the pairs)
    const bool hi = fminf(a2, a3) < fminf(a0, a1);     // the zero falls in the second pair
    const uint32_t z = hi ? (a3 < a2 ? 3u : 2u) : (a1 < a0 ? 1u : 0u);
    const uint32_t neg = (w0 < 0.0f ? 1u : 0u) | (w1 < 0.0f ? 2u : 0u) | (w2 < 0.0f ? 4u : 0u) |
                         (w3 < 0.0f ? 8u : 0u);
    // masked sum (m0 + m1) + (m2 + m3) with the zeroed weight as +0.0: in the pair
    // holding the zero, +0.0 + the other |w| is that |w|, i.e. the pair's max
    const float s01 = hi ? a0 + a1 : fmaxf(a0, a1);
    const float s23 = hi ? fmaxf(a2, a3) : a2 + a3;
    mag = s01 + s23;
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

// granularity of what kernel 1 writes to `out`
enum QMode { kQGroup = 0, kQChannel = 1, kQTensorPartials = 2 };
// fake-quantised output of kernel 1
enum QWq { kWqNone = 0, kWqF32 = 1, kWqBF16 = 2 };

struct QProb {
    const void* W;
    uint32_t* idx;
    uint8_t* sgn;
    float* out;      // scales (group, channel) or per-row subtree sums (per-tensor)
    void* Wq;        // fake-quantised weights (group and channel scales only)
    uint16_t* dead;  // Tequila-style dead-weight plane (or null)
    float* dead_sum; // its row sums (or null)
    float eps;
    int64_t row_begin;
    int N, K;
    int w_bf16, mode, gw, wq;  // gw: words per group (group), per subtree (per-tensor)
    float D;
};

template <int MAXP>
struct QParams {
    int count;
    int64_t total_rows;
    QProb p[MAXP];
};

// Packed words, sign bytes and word sums of row n (phase 1).
template <bool kBF16>
__device__ __forceinline__ void encode_row(const QProb& pr, int64_t n, const uint8_t* ctab, float* wsum,
                                           float* dsum) {
    using L = WLoad<kBF16>;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int words = pr.K >> 5;
    const int n16 = pr.K >> 4;               // 16-weight pieces (two per word)
    const int nsteps = (n16 + 31) >> 5;      // 512 weights = 16 words = one warp-step
    const int64_t row16 = n * (int64_t)n16;
    const int64_t row_word = n * (int64_t)words;
    for (int c0 = warp; c0 < nsteps; c0 += (kQThreads / 32) * kQUnroll) {
        typename L::T v[kQUnroll];
#pragma unroll
        for (int u = 0; u < kQUnroll; ++u) {
            const int piece = (c0 + (kQThreads / 32) * u) * 32 + lane;
            v[u] = (c0 + (kQThreads / 32) * u < nsteps && piece < n16) ? L::load(pr.W, row16 + piece) : L::zero();
        }
#pragma unroll
        for (int u = 0; u < kQUnroll; ++u) {
            const int c = c0 + (kQThreads / 32) * u;
            if (c >= nsteps) continue;  // warp-uniform
            const int piece = c * 32 + lane;
            const int half = lane & 1;
            uint32_t nib = 0, sg = 0;
            float m4[4], d4[4];
            uint32_t dbits[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float w0, w1, w2, w3;
                L::block(v[u], j, w0, w1, w2, w3);
                const uint32_t code = encode4(w0, w1, w2, w3, ctab, m4[j]);
                nib |= (code & 15u) << (4 * j);
                sg |= (code >> 4) << j;
                if (pr.dead) {
                    // the zeroed weight times eps, rounded to bf16 (one fp32 product)
                    const uint32_t z = (code >> 2) & 3u;
                    const float wz = z == 0 ? w0 : z == 1 ? w1 : z == 2 ? w2 : w3;
                    dbits[j] = __bfloat16_as_ushort(__float2bfloat16_rn(pr.eps * wz));
                    d4[j] = __uint_as_float(dbits[j] << 16);
                }
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
                pr.idx[row_word + w] = word;
                pr.sgn[row_word + w] = (uint8_t)sb;
                wsum[w] = s;
            }
            if (pr.dead) {
                // the lane's 4 dead values (8 bytes), and their word sum in tree order
                if (piece < n16)
                    *reinterpret_cast<uint2*>(pr.dead + n * (int64_t)(pr.K >> 2) + 4 * (int64_t)piece) =
                        make_uint2(dbits[0] | (dbits[1] << 16), dbits[2] | (dbits[3] << 16));
                float ds = (d4[0] + d4[1]) + (d4[2] + d4[3]);
                const float od = __shfl_xor_sync(kFull, ds, 1);
                ds = half ? od + ds : ds + od;
                if (half == 0 && piece < n16) dsum[piece >> 1] = ds;
            }
        }
    }
}

template <int MAXP>
__global__ void __launch_bounds__(kQThreads) k_quantize(const __grid_constant__ QParams<MAXP> P) {
    extern __shared__ float qsm[];   // [words] word sums, [words] dead-value sums, [ngroups] scales of the row
    __shared__ uint8_t ctab[64];     // 5-bit code by (zero position, negative bits)
    __shared__ float4 tpat[32];      // the block's ternary values by 5-bit code
    for (int i = threadIdx.x; i < 64; i += kQThreads) ctab[i] = (uint8_t)code_of(i >> 4, i & 15u);
    if (threadIdx.x < 32) {
        // inverse of code_of: the kept signs in position order, the zero slot reinserted
        const uint32_t nib = threadIdx.x & 15u, g = threadIdx.x >> 4;
        const uint32_t z = nib >> 2, d1 = (nib >> 1) & 1u, d2 = nib & 1u;
        const uint32_t k3 = g | ((g ^ d1) << 1) | ((g ^ d2) << 2);
        const uint32_t negs = (k3 & ((1u << z) - 1u)) | ((k3 >> z) << (z + 1));
        float t[4];
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) t[i] = (i == z) ? 0.0f : (((negs >> i) & 1u) ? -1.0f : 1.0f);
        tpat[threadIdx.x] = make_float4(t[0], t[1], t[2], t[3]);
    }
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    int pi = 0;  // rows are visited in increasing order per CTA
    for (int64_t r = blockIdx.x; r < P.total_rows; r += gridDim.x) {
        while (pi + 1 < P.count && P.p[pi + 1].row_begin <= r) ++pi;
        const QProb& pr = P.p[pi];
        const int64_t n = r - pr.row_begin;
        const int words = pr.K >> 5;
        float* wsum = qsm;
        float* dsum = qsm + words;            // dead-value word sums (Tequila plane)
        float* srow = qsm + 2 * words;
        __syncthreads();  // the tables are ready; the previous row is done with the shared buffers
        if (pr.w_bf16)
            encode_row<true>(pr, n, ctab, wsum, dsum);
        else
            encode_row<false>(pr, n, ctab, wsum, dsum);
        __syncthreads();
        if (pr.dead_sum && warp == (kQThreads / 32) - 1) {
            const float B = warp_tree_sum(dsum, words);
            if (lane == 0) pr.dead_sum[n] = B;
        }

        if (pr.mode == kQGroup) {
            // one scale per group of gw words: upper tree levels over the word sums
            const int gw = pr.gw;
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
                } else if (gw <= 16) {
                    S = tree_sum16(v, gw);
                } else {
                    S = tree_sum_seq(v, gw);
                }
                const float a = S / pr.D;
                pr.out[n * ngroups + j] = a;
                srow[j] = a;
            }
        } else if (pr.mode == kQChannel) {
            if (warp == 0) {
                const float S = warp_tree_sum(wsum, words);
                if (lane == 0) {
                    pr.out[n] = S / pr.D;
                    srow[0] = S / pr.D;
                }
            }
        } else {
            // per-tensor: sums of the aligned 2^j-weight subtrees that tile the row
            const int nparts = words / pr.gw;
            for (int j = warp; j < nparts; j += kQThreads / 32) {
                const float S = warp_tree_sum(wsum + j * pr.gw, pr.gw);
                if (lane == 0) pr.out[n * nparts + j] = S;
            }
        }

        if (pr.wq != kWqNone) {
            // fake-quantised row t * alpha from the packed words this CTA just wrote
            __syncthreads();
            const int64_t row_word = n * (int64_t)words;
            const int bpg = pr.mode == kQGroup ? pr.gw * 8 : 0x7fffffff;  // blocks per scale domain
            const int nblocks = pr.K >> 2;
            for (int b = threadIdx.x; b < nblocks; b += kQThreads) {
                const uint32_t wd = __ldcg(pr.idx + row_word + (b >> 3));
                const uint32_t sb = __ldcg(pr.sgn + row_word + (b >> 3));
                const uint32_t code = ((wd >> (4 * (b & 7))) & 15u) | (((sb >> (b & 7)) & 1u) << 4);
                const float4 t = tpat[code];
                const float a = srow[b / bpg];
                const float4 q = make_float4(t.x * a, t.y * a, t.z * a, t.w * a);
                const int64_t e = n * (int64_t)pr.K + 4 * (int64_t)b;
                if (pr.wq == kWqF32) {
                    __stcs(reinterpret_cast<float4*>(static_cast<float*>(pr.Wq) + e), q);
                } else {
                    const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(q.x)) |
                                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(q.y)) << 16);
                    const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(q.z)) |
                                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(q.w)) << 16);
                    __stcs(reinterpret_cast<uint2*>(static_cast<uint16_t*>(pr.Wq) + e), make_uint2(lo, hi));
                }
            }
        }
    }
}

// Per-tensor finalize, one CTA per tensor: canonical tree over the tensor's
// `count` subtree sums (a power-of-two segment per thread, sequential tree,
// then xor butterflies across lanes and a fixed pairwise order across warps),
// then / D.
struct QFin {
    const float* parts;
    int64_t count;
    float D;
    float* scale;
};

template <int MAXP>
struct QFinParams {
    QFin f[MAXP];
};

template <int MAXP>
__global__ void __launch_bounds__(1024) k_tensor_scale(const __grid_constant__ QFinParams<MAXP> P) {
    __shared__ float red[32];
    const QFin& F = P.f[blockIdx.x];
    const int t = threadIdx.x;
    const int64_t count = F.count;
    const int64_t Pw = pow2_ceil64(count > 0 ? count : 1);
    const int64_t seg = Pw > 1024 ? Pw / 1024 : 1;
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
            float y = __ldcg(F.parts + lo + i);
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
        if (t == 0) *F.scale = y / F.D;
    }
}

// ---- host side ---------------------------------------------------------------

static size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// largest power of two dividing K, i.e. the subtree size that tiles both each
// row and the flattened tensor
static int64_t tensor_chunk(int64_t K) { return K & (-K); }

// per-tensor only: the subtree sums of every row, rounded up to 256 bytes (a
// batched call places each weight's sums at a 256-byte boundary)
size_t quantize_workspace_bytes(int64_t N, int64_t K, int granularity) {
    if (granularity != SHERRY_PER_TENSOR || N <= 0) return 0;
    return align256((size_t)(N * (K / tensor_chunk(K))) * sizeof(float));
}

size_t quantize_batch_workspace_bytes(const QuantizeJob* jobs, int count) {
    size_t b = 0;
    for (int i = 0; i < count; ++i)
        if (jobs[i].granularity == SHERRY_PER_TENSOR && jobs[i].N > 0)
            b += quantize_workspace_bytes(jobs[i].N, jobs[i].K, SHERRY_PER_TENSOR);
    return b;
}

static float denom(int64_t L) {
    double d = (double)L / 4.0 * 3.0;
    if (d < 1.0) d = 1.0;
    return (float)d;
}

template <int MAXP>
static int quantize_launch_t(const std::vector<QProb>& probs, int64_t rows, int sms, cudaStream_t stream) {
    static QParams<MAXP> P;
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    P.count = (int)probs.size();
    P.total_rows = rows;
    int maxw = 0, maxg = 1;
    for (int i = 0; i < P.count; ++i) {
        P.p[i] = probs[i];
        maxw = std::max(maxw, probs[i].K / 32);
        if (probs[i].mode == kQGroup) maxg = std::max(maxg, probs[i].K / 32 / probs[i].gw);
    }
    const size_t smem = (size_t)(2 * maxw + maxg) * sizeof(float);
    if (smem > 48 * 1024) {
        static PerDevice attr;
        int done = 0;
        const int st = per_device(attr, &done, [](int& v) {
            SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_quantize<MAXP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   3 * (SHERRY_MAX_K / 32) * (int)sizeof(float)));
            v = 1;
            return SHERRY_OK;
        });
        if (st) return st;
    }
    const int64_t grid = std::min<int64_t>(rows, (int64_t)sms * kQCtasPerSm);
    k_quantize<MAXP><<<(unsigned)grid, kQThreads, smem, stream>>>(P);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

template <int MAXP>
static int finalize_launch_t(const std::vector<QFin>& fins, cudaStream_t stream) {
    static QFinParams<MAXP> P;
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    for (size_t i = 0; i < fins.size(); ++i) P.f[i] = fins[i];
    k_tensor_scale<MAXP><<<(unsigned)fins.size(), 1024, 0, stream>>>(P);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

int quantize_jobs_launch(const QuantizeJob* jobs, int count, void* workspace, int sms, cudaStream_t stream) {
    std::vector<QProb> probs;
    std::vector<QFin> fins;
    std::vector<sherry_unpack_desc> tensor_wq;  // per-tensor fake-quant outputs: written from the planes
    std::vector<int> tensor_wq_f32;
    int64_t rows = 0;
    size_t ws_off = 0;
    for (int i = 0; i < count; ++i) {
        const QuantizeJob& j = jobs[i];
        if (j.granularity == SHERRY_PER_TENSOR && j.N == 0) {
            // an empty tensor: alpha = 0 / max(0, 1) = 0
            SHERRY_CUDA_CHECK(cudaMemsetAsync(j.scales, 0, sizeof(float), stream));
            continue;
        }
        if (j.N == 0) continue;
        QProb p{};
        p.W = j.W;
        p.idx = j.idx;
        p.sgn = j.sgn;
        p.Wq = j.Wq;
        p.row_begin = rows;
        p.N = (int)j.N;
        p.K = (int)j.K;
        p.w_bf16 = j.w_dtype == SHERRY_BF16;
        p.wq = j.Wq == nullptr ? kWqNone : (j.wq_dtype == SHERRY_BF16 ? kWqBF16 : kWqF32);
        p.dead = j.D;
        p.dead_sum = j.D ? j.bias : nullptr;
        p.eps = j.eps;
        if (j.granularity == SHERRY_PER_GROUP) {
            p.mode = kQGroup;
            p.gw = j.group / 32;
            p.D = denom(j.group);
            p.out = j.scales;
        } else if (j.granularity == SHERRY_PER_CHANNEL) {
            p.mode = kQChannel;
            p.D = denom(j.K);
            p.out = j.scales;
        } else {
            const int64_t c = tensor_chunk(j.K);
            p.mode = kQTensorPartials;
            p.gw = (int)(c / 32);
            p.wq = kWqNone;
            p.out = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws_off);
            fins.push_back(QFin{p.out, j.N * (j.K / c), denom(j.N * j.K), j.scales});
            ws_off += quantize_workspace_bytes(j.N, j.K, SHERRY_PER_TENSOR);
            if (j.Wq) {
                tensor_wq.push_back(sherry_unpack_desc{j.idx, j.sgn, j.scales, j.N, j.K, j.granularity, j.group,
                                                       static_cast<uint16_t*>(j.Wq)});
                tensor_wq_f32.push_back(j.wq_dtype != SHERRY_BF16);
            }
        }
        rows += j.N;
        probs.push_back(p);
    }
    int st = SHERRY_OK;
    if (!probs.empty()) {
        const size_t c = probs.size();
        st = c <= 1 ? quantize_launch_t<1>(probs, rows, sms, stream)
                    : c <= 16 ? quantize_launch_t<16>(probs, rows, sms, stream)
                              : quantize_launch_t<SHERRY_MAX_BATCH>(probs, rows, sms, stream);
        if (st) return st;
    }
    if (!fins.empty()) {
        const size_t c = fins.size();
        st = c <= 1 ? finalize_launch_t<1>(fins, stream)
                    : c <= 16 ? finalize_launch_t<16>(fins, stream) : finalize_launch_t<SHERRY_MAX_BATCH>(fins, stream);
        if (st) return st;
    }
    if (!tensor_wq.empty())
        st = unpack_launch_ex(tensor_wq.data(), tensor_wq_f32.data(), (int)tensor_wq.size(), stream, sms);
    return st;
}

}  // namespace sherry
