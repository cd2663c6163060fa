// tequila.cu -- the Tequila-style dead-weight term added to a packed linear.
//
// "Sherry, Tequila and Fairies in Python", sections 1.2 and 2.1 (UltraQuantV2,
// UltraQuantLinear): the weights that a ternary quantiser sets to zero are kept
// as B = eps * w and enter the layer as a second linear term, F.linear(ones, B)
// or F.linear(sign(x), B), added to F.linear(x, A).  With Sherry's 3:4 blocks
// the zeroed weight of block b of row n is the one the packed index marks
// (zero position z = nibble >> 2); its value eps * w, rounded to bf16, is the
// dead-weight plane D[n][b] written by the quantise kernel, and the row sums of
// D are the "ones" term.
//
//   mode 0 (ones):  Y[m][n] = Yin[m][n] + bias[n]
//   mode 1 (signs): Y[m][n] = Yin[m][n] + sum_b sign(X[m][4b + z]) * D[n][b]
//
// Yin is the fp32 output of the packed linear; Y is fp32 or bf16 (round to
// nearest even of the fp32 sum).  The sign term runs on CUDA cores: each warp
// owns one output row, lanes walk its blocks (coalesced D and index loads), the
// activations of up to 8 tokens sit in shared memory per 2048-wide K chunk, and
// each lane's sums are reduced across the warp in a fixed (xor) order, so the
// term is deterministic.  Bound: the D plane (0.5 B per weight) and the index
// plane stream from HBM once per 8 tokens.
#include "common.cuh"

#include <cuda_bf16.h>

#include <algorithm>

namespace sherry {

constexpr int kTqWarps = 8;      // output rows per CTA
constexpr int kTqTok = 8;        // tokens per pass
constexpr int kTqKc = 2048;      // K chunk of activations staged in shared memory

struct TqParams {
    const uint16_t* X;
    const uint32_t* idx;
    const uint16_t* D;
    const float* bias;
    const float* Yin;
    void* Y;
    int M, N, K, y_bf16;
};

__device__ __forceinline__ void tq_store(const TqParams& P, int64_t e, float v) {
    if (P.y_bf16)
        reinterpret_cast<__nv_bfloat16*>(P.Y)[e] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float*>(P.Y)[e] = v;
}

// mode 0: one thread per output element
__global__ void __launch_bounds__(256) k_tequila_bias(const TqParams P) {
    const int64_t total = (int64_t)P.M * P.N;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x)
        tq_store(P, e, P.Yin[e] + __ldg(P.bias + e % P.N));
}

// mode 1: warp per row n, token pass blockIdx.y (tokens kTqTok * y ..)
__global__ void __launch_bounds__(32 * kTqWarps) k_tequila_sign(const TqParams P) {
    __shared__ __align__(16) uint16_t xs[kTqTok][kTqKc];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = blockIdx.x * kTqWarps + warp;
    const int m0 = blockIdx.y * kTqTok;
    const int words = P.K >> 5, nb = P.K >> 2;
    float acc[kTqTok];
#pragma unroll
    for (int m = 0; m < kTqTok; ++m) acc[m] = 0.0f;
    for (int kc = 0; kc < P.K; kc += kTqKc) {
        const int kl = min(kTqKc, P.K - kc);  // a multiple of 32
        __syncthreads();
        // stage the chunk's activations of this pass's tokens (absent tokens read as 0)
        for (int i = threadIdx.x; i < kTqTok * (kTqKc / 8); i += blockDim.x) {
            const int m = i / (kTqKc / 8), c8 = i % (kTqKc / 8);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (m0 + m < P.M && 8 * c8 < kl)
                v = __ldg(reinterpret_cast<const uint4*>(P.X + (int64_t)(m0 + m) * P.K + kc) + c8);
            *reinterpret_cast<uint4*>(&xs[m][8 * c8]) = v;
        }
        __syncthreads();
        if (n < P.N) {
            const uint32_t* irow = P.idx + (int64_t)n * words;
            const uint16_t* drow = P.D + (int64_t)n * nb;
            for (int bl = lane; bl < kl / 4; bl += 32) {
                const int b = kc / 4 + bl;
                const uint32_t z = (__ldg(irow + (b >> 3)) >> (4 * (b & 7) + 2)) & 3u;
                const float d = __uint_as_float((uint32_t)__ldg(drow + b) << 16);
#pragma unroll
                for (int m = 0; m < kTqTok; ++m) {
                    const float x = __uint_as_float((uint32_t)xs[m][4 * bl + z] << 16);
                    acc[m] += x > 0.0f ? d : (x < 0.0f ? -d : 0.0f);
                }
            }
        }
    }
    if (n >= P.N) return;
#pragma unroll
    for (int m = 0; m < kTqTok; ++m)
        for (int off = 16; off >= 1; off >>= 1) acc[m] += __shfl_xor_sync(kFull, acc[m], off);
    if (lane < kTqTok && m0 + lane < P.M) {
        float a = acc[0];
#pragma unroll
        for (int m = 1; m < kTqTok; ++m)
            if (lane == m) a = acc[m];
        const int64_t e = (int64_t)(m0 + lane) * P.N + n;
        tq_store(P, e, P.Yin[e] + a);
    }
}

int tequila_term_launch(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* idx, const uint16_t* D,
                        const float* bias, int mode, const float* Yin, void* Y, int y_bf16, cudaStream_t stream) {
    if (M == 0 || N == 0) return SHERRY_OK;
    TqParams P{X, idx, D, bias, Yin, Y, (int)M, (int)N, (int)K, y_bf16};
    if (mode == 0) {
        const int64_t total = M * N;
        const int64_t blocks = std::min<int64_t>((total + 255) / 256, 148 * 16);
        k_tequila_bias<<<(unsigned)blocks, 256, 0, stream>>>(P);
    } else {
        const dim3 grid((unsigned)((N + kTqWarps - 1) / kTqWarps), (unsigned)((M + kTqTok - 1) / kTqTok));
        if (grid.y > 65535) return SHERRY_ERR_UNSUPPORTED;
        k_tequila_sign<<<grid, 32 * kTqWarps, 0, stream>>>(P);
    }
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

}  // namespace sherry
