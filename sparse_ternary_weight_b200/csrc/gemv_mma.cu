// gemv_mma.cu -- packed 3:4 ternary linear for a few tokens (2 <= M <= 8) with
// warp-level tensor-core MMAs, Y = X (T alpha)^T ("Sherry: Hardware-Efficient
// 1.25-Bit Ternary Quantization via Fine-grained Sparsification", digest: Y = X
// T alpha, alpha applied once per group).
//
// With a few tokens the layer is a stream of packed weights, each multiplied by
// only M activations.  Every warp owns 16 weight rows and walks all of K; per
// 16-wide K slice a lane expands one block of 4 weights of each of its two rows
// (rows g and g + 8, g = lane / 4) straight into the A fragment of an
// mma.sync m16n8k16 (bf16 in, fp32 out), so the expanded weights never leave
// registers.  K is permuted inside each 32-weight packed word, identically for
// both operands: in slice h (h = 0, 1) of the word, the lane with c = lane % 4
// holds fragment positions k = 2c, 2c+1, 2c+8, 2c+9, taken to be the 4
// consecutive weights of block 2c + h; its two blocks per word are then one byte
// of the packed word, and its activation fragments for both slices are the 8
// consecutive activations 8c .. 8c+7 of the word, one 16-byte load.  A block's
// bf16 {-1, 0, +1} come from two 32-entry pattern tables (weights 0, 1 and 2, 3)
// indexed by the 5-bit code; each scale group is accumulated in two independent
// MMA fp32 fragments (one per slice of the word, for instruction-level
// parallelism), which are added in a fixed order and promoted with alpha into
// fp32 registers at the group's end (per-row scales: once at the end).
//
// Grid: one CTA of 8 warps per 128 rows of one linear; any number of
// independent linears with the same M in one launch.
#include "common.cuh"
#include "lut.cuh"

#include <cuda_bf16.h>

#include <mutex>

namespace sherry {

constexpr int kHThreads = 256;  // 8 warps x 16 rows
constexpr int kHRows = 128;
constexpr int kHKStep = 128;    // K per iteration: 4 packed words per row

struct HProb {
    const uint16_t* X;
    const uint32_t* idx;
    const uint8_t* sgn;
    const float* scales;
    void* Y;
    int N, K, words;
    int row_scale, per_tensor, spr, gwords;  // gwords: packed words per scale group
    int unit_begin;
};

template <int MAXP>
struct HParams {
    int count, M, y_bf16, total_units;
    HProb p[MAXP];
};

namespace {

__device__ __forceinline__ void hmma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                     uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int MAXP>
__device__ __forceinline__ int h_locate(const HParams<MAXP>& P, int u) {
    int lo = 0, hi = P.count - 1;  // last problem with unit_begin <= u
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.p[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
}

}  // namespace

template <int NT, int MAXP>
__global__ void __launch_bounds__(kHThreads, NT == 1 ? 3 : 2) k_hmma(const __grid_constant__ HParams<MAXP> P) {
    __shared__ __align__(256) uint32_t pat[64];  // bf16 pairs: [code] weights 0, 1; [32 + code] weights 2, 3
    if (threadIdx.x < 32) {
        const uint2 e = decode_block_bf16(threadIdx.x & 15u, threadIdx.x >> 4);
        pat[threadIdx.x] = e.x;
        pat[32 + threadIdx.x] = e.y;
    }
    __syncthreads();
    const uint32_t tbl = smem_u32(pat);

    const int u = blockIdx.x;
    const HProb& pr = P.p[h_locate(P, u)];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int N = pr.N, K = pr.K, words = pr.words, M = P.M;
    const int r0 = (u - pr.unit_begin) * kHRows + warp * 16 + g, r1 = r0 + 8;
    const bool ok0 = r0 < N, ok1 = r1 < N;
    if (r0 - g >= N) return;  // the warp's 16 rows are all past the end
    const int q0 = ok0 ? r0 : N - 1, q1 = ok1 ? r1 : N - 1;
    const uint4* w0p = reinterpret_cast<const uint4*>(pr.idx + (int64_t)q0 * words);
    const uint4* w1p = reinterpret_cast<const uint4*>(pr.idx + (int64_t)q1 * words);
    const uint32_t* s0p = reinterpret_cast<const uint32_t*>(pr.sgn + (int64_t)q0 * words);
    const uint32_t* s1p = reinterpret_cast<const uint32_t*>(pr.sgn + (int64_t)q1 * words);
    // activations 8c .. 8c+7 of every word for this lane's tokens (8 t + g); tokens >= M are zero
    const uint4* xp[NT];
    bool xok[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        xok[t] = 8 * t + g < M;
        xp[t] = reinterpret_cast<const uint4*>(pr.X + (int64_t)(xok[t] ? 8 * t + g : 0) * K) + c;
    }
    // two independent MMA accumulation chains (slice h of every word: cf[h]), added
    // in a fixed order when a scale group ends
    float cf[2][NT][4], acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[t][i] = 0.0f;
            cf[0][t][i] = cf[1][t][i] = 0.0f;
        }

    const bool gsc = !pr.row_scale;
    const int spr = pr.spr, gwords = pr.gwords;
    const float* sc0 = pr.scales + (int64_t)q0 * spr;
    const float* sc1 = pr.scales + (int64_t)q1 * spr;
    int gleft = gwords, gi = 0;  // words left in the current scale group, group index
    float al0 = gsc ? __ldg(sc0) : 1.0f, al1 = gsc ? __ldg(sc1) : 1.0f;

    const int nit = K / kHKStep;
    const uint32_t bsh = 8u * (uint32_t)c, gsh = 2u * (uint32_t)c;
    uint4 wa = __ldg(w0p), wb = __ldg(w1p);
    uint32_t sa = __ldg(s0p), sb = __ldg(s1p);
    for (int it = 0; it < nit; ++it) {
        // next iteration's packed words in flight while this one is expanded
        uint4 na = wa, nb = wb;
        uint32_t nsa = sa, nsb = sb;
        if (it + 1 < nit) {
            na = __ldg(w0p + it + 1);
            nb = __ldg(w1p + it + 1);
            nsa = __ldg(s0p + it + 1);
            nsb = __ldg(s1p + it + 1);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t xa = (q == 0 ? wa.x : q == 1 ? wa.y : q == 2 ? wa.z : wa.w) >> bsh;
            const uint32_t xb = (q == 0 ? wb.x : q == 1 ? wb.y : q == 2 ? wb.z : wb.w) >> bsh;
            const uint32_t ga = sa >> (8 * q + gsh), gb = sb >> (8 * q + gsh);
            uint4 xv[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                xv[t] = make_uint4(0u, 0u, 0u, 0u);
                if (xok[t]) xv[t] = __ldg(xp[t] + (it * kHKStep + 32 * q) / 8);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // block 2c + h of the word: nibble h of byte c, sign bit h of the lane's pair
                const uint32_t ia = tbl + ((((xa >> (4 * h)) & 15u) | (((ga >> h) & 1u) << 4)) << 2);
                const uint32_t ib = tbl + ((((xb >> (4 * h)) & 15u) | (((gb >> h) & 1u) << 4)) << 2);
                uint32_t a0, a1, a2, a3;
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a0) : "r"(ia));
                asm volatile("ld.shared.u32 %0, [%1+128];" : "=r"(a2) : "r"(ia));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a1) : "r"(ib));
                asm volatile("ld.shared.u32 %0, [%1+128];" : "=r"(a3) : "r"(ib));
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    hmma(cf[h][t], a0, a1, a2, a3, h ? xv[t].z : xv[t].x, h ? xv[t].w : xv[t].y);
            }
            if (gsc && --gleft == 0) {
                // end of a scale group: promote with alpha(row, group)
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc[t][i] = fmaf(i < 2 ? al0 : al1, cf[0][t][i] + cf[1][t][i], acc[t][i]);
                        cf[0][t][i] = cf[1][t][i] = 0.0f;
                    }
                gleft = gwords;
                ++gi;
                if (gi < spr) {
                    al0 = __ldg(sc0 + gi);
                    al1 = __ldg(sc1 + gi);
                }
            }
        }
        wa = na;
        wb = nb;
        sa = nsa;
        sb = nsb;
    }
    if (!gsc) {
        const float b0 = __ldg(pr.scales + (pr.per_tensor ? 0 : q0));
        const float b1 = __ldg(pr.scales + (pr.per_tensor ? 0 : q1));
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[t][i] = (cf[0][t][i] + cf[1][t][i]) * (i < 2 ? b0 : b1);
    }
    // fragment (row g / g + 8, tokens 8 t + 2c, 2c + 1) -> Y[token][row]
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = 8 * t + 2 * c + (i & 1);
            const int n = (i < 2) ? r0 : r1;
            if (m < M && ((i < 2) ? ok0 : ok1)) {
                if (P.y_bf16)
                    reinterpret_cast<__nv_bfloat16*>(pr.Y)[(int64_t)m * N + n] = __float2bfloat16_rn(acc[t][i]);
                else
                    reinterpret_cast<float*>(pr.Y)[(int64_t)m * N + n] = acc[t][i];
            }
        }
    }
}

// ---- host side -------------------------------------------------------------------

// up to 8 tokens (one n8 tile) this kernel is the fastest few-token path on the
// 3B decode stack (M = 2, 4, 8: 0.490, 0.510, 0.566 ms per step); from 9 tokens
// on the tcgen05 kernel wins (M = 16: 0.634 vs 0.760 ms)
bool hmma_eligible(const ProbShape& s, int64_t M) {
    if (M < 2 || M > 8 || s.N == 0) return false;
    if (s.K % kHKStep != 0) return false;
    return true;  // per-group: group % 32 == 0 always holds, so groups end on word boundaries
}

template <int NT, int MAXP>
static int hmma_launch_t(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M,
                         int y_bf16, cudaStream_t stream) {
    static HParams<MAXP> P;
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    P.count = count;
    P.M = (int)M;
    P.y_bf16 = y_bf16;
    int ub = 0;
    for (int i = 0; i < count; ++i) {
        const ProbShape& s = shapes[i];
        HProb& p = P.p[i];
        p.X = descs[i].X;
        p.idx = descs[i].idx;
        p.sgn = descs[i].sgn;
        p.scales = descs[i].scales;
        p.Y = descs[i].Y;
        p.N = (int)s.N;
        p.K = (int)s.K;
        p.words = (int)(s.K / 32);
        p.row_scale = s.granularity != SHERRY_PER_GROUP;
        p.per_tensor = s.granularity == SHERRY_PER_TENSOR;
        p.spr = s.granularity == SHERRY_PER_GROUP ? (int)(s.K / s.group) : 1;
        p.gwords = s.granularity == SHERRY_PER_GROUP ? s.group / 32 : (int)(s.K / 32);
        p.unit_begin = ub;
        ub += (int)((s.N + kHRows - 1) / kHRows);
    }
    P.total_units = ub;
    if (ub == 0) return SHERRY_OK;
    k_hmma<NT, MAXP><<<ub, kHThreads, 0, stream>>>(P);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

template <int NT>
static int hmma_launch_n(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M,
                         int y_bf16, cudaStream_t stream) {
    if (count <= 1) return hmma_launch_t<NT, 1>(shapes, descs, count, M, y_bf16, stream);
    if (count <= 16) return hmma_launch_t<NT, 16>(shapes, descs, count, M, y_bf16, stream);
    return hmma_launch_t<NT, SHERRY_MAX_BATCH>(shapes, descs, count, M, y_bf16, stream);
}

int hmma_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                       cudaStream_t stream) {
    if (M > 8) return SHERRY_ERR_UNSUPPORTED;  // one n8 token tile
    return hmma_launch_n<1>(shapes, descs, count, M, y_bf16, stream);
}

}  // namespace sherry
