/*
 * sherry_ref.h -- CPU oracle for Sherry 3:4-sparse ternary quantisation.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file; only the test-suite, the smoke check and the CPU-baseline leg
 * of the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library: every definition here is written out independently from the
 * method's description.
 *
 * Sources (page titles, sections):
 *  - "Sherry, Tequila and Fairies in Python", section 1.1 Sherry Quantization:
 *    3:4 constraint (exactly 3 of every 4 consecutive weights are +-1, one is 0),
 *    the N:M quantiser (top-n magnitudes per block of m kept, sign taken,
 *    scale = sum|kept| / max(len*n/m, 1)), the granularity reshape and its
 *    error conditions, F.linear(x, w).
 *  - "Sherry: Hardware-Efficient 1.25-Bit Ternary Quantization via Fine-grained
 *    Sparsification" (English digest): greedy Sparse-AbsMean (zero the
 *    smallest |w| of the block, signs on the rest, scale = mean |kept|),
 *    C(4,3)*2^3 = 32 states = 5 bits = 1 sign bit + 4 lookup bits, Y = X T alpha,
 *    group size 128 by default.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - tie in the minimum |w|: the lowest index is zeroed;
 *  - sign(0) = +1, also for -0.0 (IEEE w >= 0);
 *  - 4-bit index = 4*z + 2*d1 + d2 (z = zero position, d1/d2 = sign of the
 *    2nd/3rd kept weight differs from the 1st), global sign bit G = sign of the
 *    1st kept weight is negative;
 *  - planes: idx uint32[N][K/32] (nibble of block j of a word at bits 4j..4j+3),
 *    sgn uint8[N][K/32] (bit j = G of block j);
 *  - scale sum in fp32 by the adjacent-pairwise tree over the scale domain padded
 *    with +0.0 to a power of two, then one IEEE division by D = L*3/4;
 *  - linear: y[m][n] = sum_k X[m][k] * Wq[n][k] accumulated in fp64, Wq = t*alpha
 *    in fp32, decoded from the packed planes.
 */
#ifndef SHERRY_REF_H
#define SHERRY_REF_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes (values fixed by the library's documented contract) */
#define SHERRY_REF_OK 0
#define SHERRY_REF_ERR_NULL 1
#define SHERRY_REF_ERR_SHAPE 2
#define SHERRY_REF_ERR_GRANULARITY 3
#define SHERRY_REF_ERR_GROUP 4
#define SHERRY_REF_ERR_DTYPE 5

/* granularity */
#define SHERRY_REF_PER_TENSOR 0
#define SHERRY_REF_PER_CHANNEL 1
#define SHERRY_REF_PER_GROUP 2

/* element types */
#define SHERRY_REF_F32 0
#define SHERRY_REF_BF16 1

/* canonical pairwise sum of v[0..L) in fp32 (padding with +0.0 to a power of two) */
float sherry_ref_pairsum(const float* v, int64_t L);

/* number of fp32 scales for a granularity (-1 on invalid arguments) */
int64_t sherry_ref_num_scales(int64_t N, int64_t K, int granularity, int group);

/* W [N][K] row-major, fp32 or bf16 bits.  Outputs are overwritten entirely. */
int sherry_ref_quantize_pack(const void* W, int w_dtype, int64_t N, int64_t K,
                             int granularity, int group,
                             uint32_t* idx, uint8_t* sgn, float* scales);

/* dense fp32 Wq[n][k] = t[n][k] * alpha, decoded from the planes only */
int sherry_ref_unpack_f32(const uint32_t* idx, const uint8_t* sgn, const float* scales,
                          int64_t N, int64_t K, int granularity, int group, float* Wq);

/* dense bf16 (bits) = round-to-nearest-even(t * alpha) */
int sherry_ref_unpack_bf16(const uint32_t* idx, const uint8_t* sgn, const float* scales,
                           int64_t N, int64_t K, int granularity, int group, uint16_t* Wb);

/* Y[m][n] (fp64) for the token rows listed in rows[0..n_rows) of X (bf16 bits,
 * [M][K] row-major); Y is [n_rows][N].  rows == NULL means all M rows. */
int sherry_ref_linear(const uint16_t* X, int64_t M, const int64_t* rows, int64_t n_rows,
                      const uint32_t* idx, const uint8_t* sgn, const float* scales,
                      int64_t N, int64_t K, int granularity, int group, double* Y);

/* The quantiser's forward output ("Sherry, Tequila and Fairies in Python",
 * section 1.1, SherryNMQuant.forward): the masked weight's signs times the
 * scale of their domain, computed directly from W (block argmin -> mask, signs,
 * pairwise sums of the kept |w|, one division) without packing.  Wq fp32
 * [N][K] (zeroed positions +0.0); Wb (optional, may be NULL) receives
 * round-to-nearest-even bf16 bits of Wq. */
int sherry_ref_fake_quant(const void* W, int w_dtype, int64_t N, int64_t K, int granularity, int group,
                          float* Wq, uint16_t* Wb);

/* Tequila-style dead-weight term on Sherry's weights ("Sherry, Tequila and
 * Fairies in Python", sections 1.2 and 2.1: UltraQuantV2 keeps the weights the
 * ternary quantiser sets to zero as B = eps * w, and UltraQuantLinear adds
 * F.linear(ones, B) -- or F.linear(sign(x), B) -- to F.linear(x, A)).  Here the
 * zeroed weights are Sherry's: the smallest |w| of every block of 4.
 * D [N][K/4] bf16 bits: round-to-nearest-even of the fp32 product eps * w at the
 * zeroed position of each block (B cast to the activations' bf16, as the page
 * does before the linear); bias [N] (optional): the canonical pairwise fp32 sum
 * of D[n][*] as fp32 values, i.e. F.linear(ones, B). */
int sherry_ref_tequila_dead(const void* W, int w_dtype, int64_t N, int64_t K, float eps, uint16_t* D, float* bias);

/* The term added to Y [M][N] (fp64): mode 0 (ones): T[m][n] = bias[n]; mode 1
 * (signs of the activations): T[m][n] = sum_b sign(x[m][4b + z(n, b)]) * D[n][b],
 * sign(0) = 0 as torch.sign, z the zero position of block b in the idx plane. */
int sherry_ref_tequila_term(const uint16_t* X, int64_t M, const uint32_t* idx, const uint16_t* D,
                            const float* bias, int64_t N, int64_t K, int mode, double* T);

/* Arenas, the annealed residual of Sherry's training ("Sherry: Hardware-Efficient
 * 1.25-Bit Ternary Quantization via Fine-grained Sparsification", digest
 * paragraph on Arenas: Y = X T alpha + lambda_t X W, lambda_t decayed to 0 with a
 * cosine, gone at inference).  Y [n_rows][N] fp64 for all token rows of X (bf16
 * bits [M][K]); Wd is the latent weight as bf16 bits [N][K]; the two products are
 * accumulated in fp64 and combined as y = yT + lambda * yW. */
int sherry_ref_arenas_linear(const uint16_t* X, int64_t M, const uint32_t* idx, const uint8_t* sgn,
                             const float* scales, const uint16_t* Wd, float lambda, int64_t N, int64_t K,
                             int granularity, int group, double* Y);
/* lambda_t = lambda0 * (1 + cos(pi * min(step, total) / total)) / 2 (cosine decay
 * from lambda0 at step 0 to 0 at step total; lambda0 for total <= 0) */
double sherry_ref_arenas_lambda(int64_t step, int64_t total, double lambda0);

/* number of threads the build uses (1 unless built with OpenMP) */
int sherry_ref_threads(void);

#ifdef __cplusplus
}
#endif
#endif
