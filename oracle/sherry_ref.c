/*
 * sherry_ref.c -- plain, slow, single-pass CPU oracle for Sherry 3:4-sparse
 * ternary quantise+pack, unpack and the packed linear layer.
 *
 * TEST INFRASTRUCTURE ONLY: used by the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark, never by the product path.  It shares
 * nothing with the CUDA library.  Build: gcc -std=c99 -O2 -fno-fast-math
 * -ffp-contract=off (optionally -fopenmp, which only splits independent rows
 * across threads and never changes a result).
 *
 * Every function follows the method's statement step by step; see the header
 * for the passages and for the readings taken where the pages are silent.
 */
#include "sherry_ref.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int sherry_ref_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static float bf16_bits_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* round-to-nearest-even fp32 -> bf16 (inputs here are finite) */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* ---- argument checks: the pages' quantiser rejects a non-2D weight, an inner
 * dimension that is not a multiple of the block (here the 32-weight word of the
 * layout), a non-positive group or one that does not divide the row, and an
 * unknown granularity. ---- */
static int check_shape(int64_t N, int64_t K) {
    if (N < 0 || K <= 0 || (K % 32) != 0) return SHERRY_REF_ERR_SHAPE;
    return SHERRY_REF_OK;
}

static int check_gran(int64_t K, int granularity, int group) {
    if (granularity == SHERRY_REF_PER_TENSOR || granularity == SHERRY_REF_PER_CHANNEL)
        return SHERRY_REF_OK;
    if (granularity != SHERRY_REF_PER_GROUP) return SHERRY_REF_ERR_GRANULARITY;
    if (group <= 0 || (group % 32) != 0 || (K % group) != 0) return SHERRY_REF_ERR_GROUP;
    return SHERRY_REF_OK;
}

int64_t sherry_ref_num_scales(int64_t N, int64_t K, int granularity, int group) {
    if (check_shape(N, K) != SHERRY_REF_OK) return -1;
    if (check_gran(K, granularity, group) != SHERRY_REF_OK) return -1;
    if (granularity == SHERRY_REF_PER_TENSOR) return 1;
    if (granularity == SHERRY_REF_PER_CHANNEL) return N;
    return N * (K / group);
}

/* scale index of weight (n, k) */
static int64_t scale_index(int64_t n, int64_t k, int64_t K, int granularity, int group) {
    if (granularity == SHERRY_REF_PER_TENSOR) return 0;
    if (granularity == SHERRY_REF_PER_CHANNEL) return n;
    return n * (K / group) + k / group;
}

/* ---- canonical pairwise sum: pad to P = 2^ceil(log2 L) with +0.0, then
 * repeatedly replace v[i] by v[2i] + v[2i+1] (fp32, round to nearest even). ---- */
float sherry_ref_pairsum(const float* v, int64_t L) {
    if (L <= 0) return 0.0f;
    int64_t P = 1;
    while (P < L) P *= 2;
    float* buf = (float*)malloc((size_t)P * sizeof(float));
    if (!buf) abort();
    for (int64_t i = 0; i < P; ++i) buf[i] = (i < L) ? v[i] : 0.0f;
    while (P > 1) {
        int64_t h = P / 2;
        for (int64_t i = 0; i < h; ++i) buf[i] = buf[2 * i] + buf[2 * i + 1];
        P = h;
    }
    float r = buf[0];
    free(buf);
    return r;
}

/* ---- one block of 4: greedy Sparse-AbsMean.
 * The weight with the smallest |w| is zeroed (first index on ties), the three
 * kept weights keep their signs (w >= 0 -> +1).  Code: z = zero position,
 * p0 < p1 < p2 the kept positions, G = [s(p0) = -1], d1 = [s(p1) != s(p0)],
 * d2 = [s(p2) != s(p0)], nibble = 4z + 2 d1 + d2.  The masked magnitudes are
 * |w| at kept positions and +0.0 at z. ---- */
static void encode_block(const float w[4], unsigned* nibble, unsigned* gbit, float mag[4]) {
    float a[4];
    int s[4];
    for (int i = 0; i < 4; ++i) {
        a[i] = fabsf(w[i]);
        s[i] = (w[i] >= 0.0f) ? 1 : -1;
    }
    int z = 0;
    for (int i = 1; i < 4; ++i)
        if (a[i] < a[z]) z = i;
    int p[3], c = 0;
    for (int i = 0; i < 4; ++i)
        if (i != z) p[c++] = i;
    unsigned G = (s[p[0]] < 0) ? 1u : 0u;
    unsigned d1 = (s[p[1]] != s[p[0]]) ? 1u : 0u;
    unsigned d2 = (s[p[2]] != s[p[0]]) ? 1u : 0u;
    *nibble = 4u * (unsigned)z + 2u * d1 + d2;
    *gbit = G;
    for (int i = 0; i < 4; ++i) mag[i] = (i == z) ? 0.0f : a[i];
}

/* inverse of encode_block on the ternary values: t[i] in {-1, 0, +1} */
static void decode_block(unsigned nibble, unsigned gbit, int t[4]) {
    int z = (int)(nibble >> 2);
    int d1 = (int)((nibble >> 1) & 1u);
    int d2 = (int)(nibble & 1u);
    int first = gbit ? -1 : 1;
    int p[3], c = 0;
    for (int i = 0; i < 4; ++i)
        if (i != z) p[c++] = i;
    t[z] = 0;
    t[p[0]] = first;
    t[p[1]] = d1 ? -first : first;
    t[p[2]] = d2 ? -first : first;
}

int sherry_ref_quantize_pack(const void* W, int w_dtype, int64_t N, int64_t K,
                             int granularity, int group,
                             uint32_t* idx, uint8_t* sgn, float* scales) {
    int st = check_shape(N, K);
    if (st) return st;
    st = check_gran(K, granularity, group);
    if (st) return st;
    if (w_dtype != SHERRY_REF_F32 && w_dtype != SHERRY_REF_BF16) return SHERRY_REF_ERR_DTYPE;
    if (N > 0 && (!W || !idx || !sgn)) return SHERRY_REF_ERR_NULL;
    if (!scales) return SHERRY_REF_ERR_NULL;

    const int64_t words = K / 32;
    /* masked magnitudes of the whole tensor, row-major */
    float* mag = (float*)malloc((size_t)(N * K > 0 ? N * K : 1) * sizeof(float));
    if (!mag) abort();

#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t w = 0; w < words; ++w) {
            idx[n * words + w] = 0u;
            sgn[n * words + w] = 0u;
        }
        for (int64_t b = 0; b < K / 4; ++b) {
            float wv[4];
            for (int i = 0; i < 4; ++i) {
                int64_t off = n * K + 4 * b + i;
                wv[i] = (w_dtype == SHERRY_REF_F32) ? ((const float*)W)[off]
                                                    : bf16_bits_to_f32(((const uint16_t*)W)[off]);
            }
            unsigned nib, g;
            encode_block(wv, &nib, &g, &mag[n * K + 4 * b]);
            idx[n * words + b / 8] |= (uint32_t)nib << (4 * (b % 8));
            sgn[n * words + b / 8] |= (uint8_t)(g << (b % 8));
        }
    }

    /* scale = PairSum(masked |w| over the domain) / D, D = max(L * 3/4, 1) */
    if (granularity == SHERRY_REF_PER_TENSOR) {
        int64_t L = N * K;
        float S = sherry_ref_pairsum(mag, L);
        double Dd = (double)L / 4.0 * 3.0;
        if (Dd < 1.0) Dd = 1.0;
        scales[0] = S / (float)Dd;
    } else if (granularity == SHERRY_REF_PER_CHANNEL) {
        float D = (float)((double)K / 4.0 * 3.0);
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
        for (int64_t n = 0; n < N; ++n) scales[n] = sherry_ref_pairsum(&mag[n * K], K) / D;
    } else {
        const int64_t G = K / group;
        float D = (float)((double)group / 4.0 * 3.0);
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < G; ++j)
                scales[n * G + j] = sherry_ref_pairsum(&mag[n * K + j * group], group) / D;
    }
    free(mag);
    return SHERRY_REF_OK;
}

/* ---- forward output of the quantiser: mask the smallest |w| of every block,
 * keep the signs (w >= 0 -> +1), scale = PairSum(masked |w| over the domain)
 * / max(L * 3/4, 1), output sign * mask * scale.  No packing is involved. ---- */
int sherry_ref_fake_quant(const void* W, int w_dtype, int64_t N, int64_t K, int granularity, int group,
                          float* Wq, uint16_t* Wb) {
    int st = check_shape(N, K);
    if (st) return st;
    st = check_gran(K, granularity, group);
    if (st) return st;
    if (w_dtype != SHERRY_REF_F32 && w_dtype != SHERRY_REF_BF16) return SHERRY_REF_ERR_DTYPE;
    if (N > 0 && (!W || !Wq)) return SHERRY_REF_ERR_NULL;

    float* mag = (float*)malloc((size_t)(N * K > 0 ? N * K : 1) * sizeof(float));
    int8_t* sgn = (int8_t*)malloc((size_t)(N * K > 0 ? N * K : 1));
    if (!mag || !sgn) abort();
    /* mask and signs, block by block */
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < K / 4; ++b) {
            float wv[4];
            for (int i = 0; i < 4; ++i) {
                int64_t off = n * K + 4 * b + i;
                wv[i] = (w_dtype == SHERRY_REF_F32) ? ((const float*)W)[off]
                                                    : bf16_bits_to_f32(((const uint16_t*)W)[off]);
            }
            unsigned nib, g;
            encode_block(wv, &nib, &g, &mag[n * K + 4 * b]);
            int z = (int)(nib >> 2);
            for (int i = 0; i < 4; ++i)
                sgn[n * K + 4 * b + i] = (int8_t)((i == z) ? 0 : ((wv[i] >= 0.0f) ? 1 : -1));
        }
    }
    /* one scale per domain, then sign * scale */
    if (granularity == SHERRY_REF_PER_TENSOR) {
        const int64_t L = N * K;
        const double kept = 3.0 * (double)L / 4.0; /* D = max(L * 3/4, 1) */
        float a = sherry_ref_pairsum(mag, L) / (float)(kept < 1.0 ? 1.0 : kept);
        for (int64_t i = 0; i < N * K; ++i) Wq[i] = (float)sgn[i] * a;
    } else {
        const int64_t L = (granularity == SHERRY_REF_PER_CHANNEL) ? K : group;
        const float D = (float)((double)L / 4.0 * 3.0);
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < K / L; ++j) {
                float a = sherry_ref_pairsum(&mag[n * K + j * L], L) / D;
                for (int64_t k = j * L; k < j * L + L; ++k) Wq[n * K + k] = (float)sgn[n * K + k] * a;
            }
    }
    if (Wb)
        for (int64_t i = 0; i < N * K; ++i) Wb[i] = f32_to_bf16_rne(Wq[i]);
    free(mag);
    free(sgn);
    return SHERRY_REF_OK;
}

/* ---- Tequila-style dead-weight term: the zeroed weight of every block, times
 * eps, rounded to bf16; its row sums for the "ones" input. ---- */
int sherry_ref_tequila_dead(const void* W, int w_dtype, int64_t N, int64_t K, float eps, uint16_t* D, float* bias) {
    int st = check_shape(N, K);
    if (st) return st;
    if (w_dtype != SHERRY_REF_F32 && w_dtype != SHERRY_REF_BF16) return SHERRY_REF_ERR_DTYPE;
    if (N > 0 && (!W || !D)) return SHERRY_REF_ERR_NULL;
    const int64_t nb = K / 4;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n) {
        float* dv = (float*)malloc((size_t)nb * sizeof(float));
        if (!dv) abort();
        for (int64_t b = 0; b < nb; ++b) {
            float wv[4], mag[4];
            for (int i = 0; i < 4; ++i) {
                int64_t off = n * K + 4 * b + i;
                wv[i] = (w_dtype == SHERRY_REF_F32) ? ((const float*)W)[off]
                                                    : bf16_bits_to_f32(((const uint16_t*)W)[off]);
            }
            unsigned nib, g;
            encode_block(wv, &nib, &g, mag);
            const float dead = eps * wv[nib >> 2];
            D[n * nb + b] = f32_to_bf16_rne(dead);
            dv[b] = bf16_bits_to_f32(D[n * nb + b]);
        }
        if (bias) bias[n] = sherry_ref_pairsum(dv, nb);
        free(dv);
    }
    return SHERRY_REF_OK;
}

int sherry_ref_tequila_term(const uint16_t* X, int64_t M, const uint32_t* idx, const uint16_t* D,
                            const float* bias, int64_t N, int64_t K, int mode, double* T) {
    int st = check_shape(N, K);
    if (st) return st;
    if (M < 0 || (mode != 0 && mode != 1)) return SHERRY_REF_ERR_SHAPE;
    if (M > 0 && N > 0 && (!T || (mode == 0 && !bias) || (mode == 1 && (!X || !idx || !D))))
        return SHERRY_REF_ERR_NULL;
    const int64_t words = K / 32, nb = K / 4;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            if (mode == 0) {
                acc = (double)bias[n];
            } else {
                for (int64_t b = 0; b < nb; ++b) {
                    const unsigned z = (idx[n * words + b / 8] >> (4 * (b % 8) + 2)) & 3u;
                    const float x = bf16_bits_to_f32(X[m * K + 4 * b + z]);
                    const double sx = (x > 0.0f) ? 1.0 : ((x < 0.0f) ? -1.0 : 0.0);
                    acc += sx * (double)bf16_bits_to_f32(D[n * nb + b]);
                }
            }
            T[m * N + n] = acc;
        }
    return SHERRY_REF_OK;
}

/* ---- Arenas: the quantised product plus lambda times the latent-weight product ---- */
double sherry_ref_arenas_lambda(int64_t step, int64_t total, double lambda0) {
    if (total <= 0) return lambda0;
    double s = (double)(step < 0 ? 0 : (step > total ? total : step));
    return lambda0 * 0.5 * (1.0 + cos(3.14159265358979323846 * s / (double)total));
}

/* ternary value of weight (n, k) decoded from the planes */
static int ternary_at(const uint32_t* idx, const uint8_t* sgn, int64_t n, int64_t k, int64_t K) {
    int64_t words = K / 32;
    int64_t b = k / 4;
    unsigned nib = (idx[n * words + b / 8] >> (4 * (b % 8))) & 0xFu;
    unsigned g = (sgn[n * words + b / 8] >> (b % 8)) & 1u;
    int t[4];
    decode_block(nib, g, t);
    return t[k % 4];
}

static int check_planes(const uint32_t* idx, const uint8_t* sgn, const float* scales,
                        int64_t N, int64_t K, int granularity, int group) {
    int st = check_shape(N, K);
    if (st) return st;
    st = check_gran(K, granularity, group);
    if (st) return st;
    if (N > 0 && (!idx || !sgn || !scales)) return SHERRY_REF_ERR_NULL;
    return SHERRY_REF_OK;
}

int sherry_ref_unpack_f32(const uint32_t* idx, const uint8_t* sgn, const float* scales,
                          int64_t N, int64_t K, int granularity, int group, float* Wq) {
    int st = check_planes(idx, sgn, scales, N, K, granularity, group);
    if (st) return st;
    if (N > 0 && !Wq) return SHERRY_REF_ERR_NULL;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            Wq[n * K + k] = (float)ternary_at(idx, sgn, n, k, K) *
                            scales[scale_index(n, k, K, granularity, group)];
    return SHERRY_REF_OK;
}

int sherry_ref_unpack_bf16(const uint32_t* idx, const uint8_t* sgn, const float* scales,
                           int64_t N, int64_t K, int granularity, int group, uint16_t* Wb) {
    int st = check_planes(idx, sgn, scales, N, K, granularity, group);
    if (st) return st;
    if (N > 0 && !Wb) return SHERRY_REF_ERR_NULL;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            float v = (float)ternary_at(idx, sgn, n, k, K) *
                      scales[scale_index(n, k, K, granularity, group)];
            Wb[n * K + k] = f32_to_bf16_rne(v);
        }
    return SHERRY_REF_OK;
}

int sherry_ref_arenas_linear(const uint16_t* X, int64_t M, const uint32_t* idx, const uint8_t* sgn,
                             const float* scales, const uint16_t* Wd, float lambda, int64_t N, int64_t K,
                             int granularity, int group, double* Y) {
    int st = check_planes(idx, sgn, scales, N, K, granularity, group);
    if (st) return st;
    if (M < 0) return SHERRY_REF_ERR_SHAPE;
    if (M > 0 && N > 0 && (!X || !Wd || !Y)) return SHERRY_REF_ERR_NULL;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double yt = 0.0, yw = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                const double x = (double)bf16_bits_to_f32(X[m * K + k]);
                yt += x * (double)((float)ternary_at(idx, sgn, n, k, K) *
                                   scales[scale_index(n, k, K, granularity, group)]);
                yw += x * (double)bf16_bits_to_f32(Wd[n * K + k]);
            }
            Y[m * N + n] = yt + (double)lambda * yw;
        }
    }
    return SHERRY_REF_OK;
}

int sherry_ref_linear(const uint16_t* X, int64_t M, const int64_t* rows, int64_t n_rows,
                      const uint32_t* idx, const uint8_t* sgn, const float* scales,
                      int64_t N, int64_t K, int granularity, int group, double* Y) {
    int st = check_planes(idx, sgn, scales, N, K, granularity, group);
    if (st) return st;
    if (M < 0) return SHERRY_REF_ERR_SHAPE;
    if (!rows) n_rows = M;
    if (n_rows < 0) return SHERRY_REF_ERR_SHAPE;
    if (n_rows > 0 && N > 0 && (!X || !Y)) return SHERRY_REF_ERR_NULL;
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t m = rows ? rows[r] : r;
        if (m < 0 || m >= M) return SHERRY_REF_ERR_SHAPE;
    }
    /* dequantised weight row by row: Wq[n][k] = t * alpha (fp32, exact) */
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n) {
        float* wrow = (float*)malloc((size_t)K * sizeof(float));
        if (!wrow) abort();
        for (int64_t k = 0; k < K; ++k)
            wrow[k] = (float)ternary_at(idx, sgn, n, k, K) *
                      scales[scale_index(n, k, K, granularity, group)];
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t m = rows ? rows[r] : r;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)bf16_bits_to_f32(X[m * K + k]) * (double)wrow[k];
            Y[r * N + n] = acc;
        }
        free(wrow);
    }
    return SHERRY_REF_OK;
}
