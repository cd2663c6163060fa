// gemv.cu -- packed 3:4 ternary linear for few tokens (decode), Y = X (T alpha)^T.
//
// "Sherry: Hardware-Efficient 1.25-Bit Ternary Quantization via Fine-grained
// Sparsification" (digest paragraph on inference): lookup tables are built from
// the activations online, the packed weights index them, the lookups are
// accumulated and the scale is applied afterwards.  The 5-bit block code is a
// sign bit plus 4 lookup bits, so one table of 32 fp32 entries per block of 4
// activations covers every state:
//     entry[16 G + 4 z + 2 d1 + d2] = (-1)^G (x_p0 + (-1)^d1 x_p1 + (-1)^d2 x_p2)
// where p0 < p1 < p2 are the positions other than z.
//
// B200 mapping.  A CTA (8 warps) owns R = 32*WR output rows and a K range; it
// builds the tables of one K sub-slice in shared memory (one table per thread),
// then every lane walks ONE row: all 32 lanes of a warp read the same table, so
// each lookup is a single conflict-free LDS (table base 128-byte... padded to
// 144 B so that the build's 16-byte stores rotate over the banks).  Per packed
// word (8 blocks) the nibbles and sign bits are spread into two byte-vectors
// (even / odd blocks) whose bytes are 4*code; one PRMT per block merges a byte
// with the table base into the LDS address.  Accumulation is fp32; alpha is
// applied once per word, step, or row.  No multiplies touch the weights.
//
// K may be split across CTAs (split-K): each CTA stores its partial row sums in
// the workspace, and the last CTA to arrive (an atomic ticket, no waiting) adds
// the partials in split order and writes Y, so results are deterministic.
#include "common.cuh"
#include "lut.cuh"

#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <vector>

namespace sherry {

constexpr int kLThreads = 256;
constexpr int kLutTables = 256;              // tables per CTA (= threads)
constexpr int kLutBytes = kLutTables * kTab; // 36864
constexpr int kLutSmem = kLutBytes + 256;    // + alignment slack

enum LMode { kModeRow = 0, kModeStep = 1, kModeWord = 2, kModeGen = 3 };

struct LinProb {
    const uint16_t* X;
    const uint32_t* idx;
    const uint8_t* sgn;
    const float* scales;
    void* Y;
    float* part;      // split-K partials (S > 1)
    int* cnt;         // split-K tickets (S > 1)
    int N, K;
    int mode;
    int row_scale;    // 1: alpha per row (channel) or tensor, applied at the end
    int per_tensor;
    int gw;           // words per group (per-group)
    int gw_shift;     // log2(gw) or -1
    int spr;          // scales per row
    int S;            // K splits
    int wps;          // words per split
    int n_rt;         // row tiles
    int n_pass;       // token passes
    int tile_begin;
};

template <int MAXP>
struct LinParams {
    int count;
    int M;
    int y_bf16;
    int total_tiles;
    LinProb p[MAXP];
};

template <int MT, int WR, int MAXP>
__global__ void __launch_bounds__(kLThreads, 2) k_lut_linear(const __grid_constant__ LinParams<MAXP> P) {
    constexpr int WK = 8 / WR;
    constexpr int R = 32 * WR;
    constexpr int KSB = kLutTables / MT;  // blocks per sub-slice
    constexpr int KSW = KSB / 8;          // words per sub-slice
    constexpr int TSTRIDE = KSB * kTab;   // bytes between tokens' tables
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int s_last;
    const uint32_t lut = (smem_u32(smem_raw) + 255u) & ~255u;
    float* red = reinterpret_cast<float*>(smem_raw + (lut - smem_u32(smem_raw)));

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int wr = warp % WR;
    const int kw = warp / WR;

    int pi = 0;  // problem cursor: tiles are visited in increasing order
    for (int t = blockIdx.x; t < P.total_tiles; t += gridDim.x) {
        while (pi + 1 < P.count && P.p[pi + 1].tile_begin <= t) ++pi;
        const LinProb& pr = P.p[pi];
        int local = t - pr.tile_begin;
        const int s = local % pr.S;
        local /= pr.S;
        const int rt = local % pr.n_rt;
        const int pass = local / pr.n_rt;
        const int m0 = pass * MT;
        const int M = P.M;
        const int N = pr.N, K = pr.K;
        const int words = K >> 5;
        const int rloc = wr * 32 + lane;
        const int n = rt * R + rloc;
        const bool row_ok = n < N;
        const int w_begin = s * pr.wps;
        const int w_end = min(words, w_begin + pr.wps);
        const int64_t row_word = (int64_t)(row_ok ? n : 0) * words;
        const uint32_t* idxr = pr.idx + row_word;
        const uint8_t* sgnr = pr.sgn + row_word;
        const float* scr = pr.scales + (int64_t)(row_ok ? n : 0) * pr.spr;

        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.0f;

        for (int sub = w_begin; sub < w_end; sub += KSW) {
            const int sub_end = min(w_end, sub + KSW);
            __syncthreads();  // previous tables no longer read
            {
                const int ml = tid / KSB;
                const int bl = tid % KSB;
                const int b = sub * 8 + bl;
                const int m = m0 + ml;
                if (b < sub_end * 8 && m < M) {
                    const uint2 xb = __ldg(reinterpret_cast<const uint2*>(pr.X + (int64_t)m * K) + b);
                    build_table(lut + (uint32_t)(ml * TSTRIDE + bl * kTab), xb);
                }
            }
            __syncthreads();
            const int nw = sub_end - sub;
            if (pr.mode != kModeGen) {
                // 4-word steps (K % 128 == 0); step si of this sub-slice goes to warp kw == si % WK
                for (int si = kw; si * 4 < nw; si += WK) {
                    const int wg = sub + si * 4;
                    uint4 wq = make_uint4(0u, 0u, 0u, 0u);
                    uint32_t sq = 0u;
                    if (row_ok) {
                        wq = __ldcs(reinterpret_cast<const uint4*>(idxr + wg));
                        sq = __ldcs(reinterpret_cast<const uint32_t*>(sgnr + wg));
                    }
                    const uint32_t base = lut + (uint32_t)(si * 32 * kTab);
                    float ws[4][MT];
                    word_lookups<MT>(wq.x, sq & 0xffu, base, 0, TSTRIDE, ws[0]);
                    word_lookups<MT>(wq.y, (sq >> 8) & 0xffu, base, 8, TSTRIDE, ws[1]);
                    word_lookups<MT>(wq.z, (sq >> 16) & 0xffu, base, 16, TSTRIDE, ws[2]);
                    word_lookups<MT>(wq.w, sq >> 24, base, 24, TSTRIDE, ws[3]);
                    if (pr.mode == kModeRow) {
#pragma unroll
                        for (int m = 0; m < MT; ++m) acc[m] += (ws[0][m] + ws[1][m]) + (ws[2][m] + ws[3][m]);
                    } else if (pr.mode == kModeStep) {
                        const float a = row_ok ? __ldg(scr + (wg >> pr.gw_shift)) : 0.0f;
#pragma unroll
                        for (int m = 0; m < MT; ++m)
                            acc[m] = fmaf(a, (ws[0][m] + ws[1][m]) + (ws[2][m] + ws[3][m]), acc[m]);
                    } else {  // kModeWord: gw is 1 or 2
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float a = row_ok ? __ldg(scr + ((wg + q) >> pr.gw_shift)) : 0.0f;
#pragma unroll
                            for (int m = 0; m < MT; ++m) acc[m] = fmaf(a, ws[q][m], acc[m]);
                        }
                    }
                }
            } else {
                // generic: one word per step, any K % 32 == 0 and any group
                for (int si = kw; si < nw; si += WK) {
                    const int wg = sub + si;
                    uint32_t w = 0u, sb = 0u;
                    if (row_ok) {
                        w = __ldcs(idxr + wg);
                        sb = __ldcs(sgnr + wg);
                    }
                    const uint32_t base = lut + (uint32_t)((si & ~3) * 8 * kTab);
                    float ws[MT];
                    word_lookups<MT>(w, sb, base, (si & 3) * 8, TSTRIDE, ws);
                    if (pr.row_scale) {
#pragma unroll
                        for (int m = 0; m < MT; ++m) acc[m] += ws[m];
                    } else {
                        const float a = row_ok ? __ldg(scr + wg / pr.gw) : 0.0f;
#pragma unroll
                        for (int m = 0; m < MT; ++m) acc[m] = fmaf(a, ws[m], acc[m]);
                    }
                }
            }
        }

        // combine the WK warps that share these rows (fixed order)
        if (WK > 1) {
            __syncthreads();
#pragma unroll
            for (int m = 0; m < MT; ++m) red[(kw * MT + m) * R + rloc] = acc[m];
            __syncthreads();
            if (kw == 0) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float v = red[m * R + rloc];
                    for (int q = 1; q < WK; ++q) v += red[(q * MT + m) * R + rloc];
                    acc[m] = v;
                }
            }
        }
        if (pr.row_scale && kw == 0 && row_ok) {
            const float a = __ldg(pr.scales + (pr.per_tensor ? 0 : n));
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] *= a;
        }

        if (pr.S == 1) {
            if (kw == 0 && row_ok) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m0 + m < M) {
                        const int64_t o = (int64_t)(m0 + m) * N + n;
                        if (P.y_bf16)
                            reinterpret_cast<__nv_bfloat16*>(pr.Y)[o] = __float2bfloat16_rn(acc[m]);
                        else
                            reinterpret_cast<float*>(pr.Y)[o] = acc[m];
                    }
                }
            }
        } else {
            const int slot = pass * pr.n_rt + rt;
            float* part = pr.part + (int64_t)slot * pr.S * MT * R;
            if (kw == 0) {
#pragma unroll
                for (int m = 0; m < MT; ++m) __stcg(part + ((int64_t)s * MT + m) * R + rloc, acc[m]);
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) s_last = (atomicAdd(pr.cnt + slot, 1) == pr.S - 1);
            __syncthreads();
            if (s_last) {
                __threadfence();
                for (int e = tid; e < MT * R; e += kLThreads) {
                    const int m = e / R, r = e % R;
                    const int nn = rt * R + r;
                    if (nn < N && m0 + m < M) {
                        float v = __ldcg(part + (int64_t)m * R + r);
                        for (int q = 1; q < pr.S; ++q) v += __ldcg(part + ((int64_t)q * MT + m) * R + r);
                        const int64_t o = (int64_t)(m0 + m) * N + nn;
                        if (P.y_bf16)
                            reinterpret_cast<__nv_bfloat16*>(pr.Y)[o] = __float2bfloat16_rn(v);
                        else
                            reinterpret_cast<float*>(pr.Y)[o] = v;
                    }
                }
                if (tid == 0) pr.cnt[slot] = 0;  // leave the ticket zeroed for the next call
            }
        }
    }
}

// ---- host side -------------------------------------------------------------------

struct DevInfo {
    int sms = 148;
};

static int tokens_per_pass(int64_t M) { return M <= 1 ? 1 : (M <= 2 ? 2 : 4); }

// make_plan splits K only with 64-row tiles (WR = 2: 256-row tiles already give
// at least the target of 2 CTAs per SM), and then gives one problem fewer than
// twice the target tiles of at most 4 tokens: the no-workspace entry point's
// fixed scratch holds that on up to 224 SMs.
static_assert(kTicketBytes + (size_t)2 * (2 * 224) * 4 * 64 * sizeof(float) <= SHERRY_NOALLOC_SCRATCH_BYTES,
              "no-workspace scratch too small for the general lookup-table plan");

struct Plan {
    int MT, WR;
    std::vector<LinProb> probs;
    int total_tiles = 0;
    size_t ws_bytes = 0;
};

static void fill_mode(LinProb& p, const ProbShape& s) {
    const bool vec4 = (s.K % 128) == 0;
    p.row_scale = s.granularity != SHERRY_PER_GROUP;
    p.per_tensor = s.granularity == SHERRY_PER_TENSOR;
    p.gw = s.granularity == SHERRY_PER_GROUP ? s.group / 32 : 0;
    p.gw_shift = s.granularity == SHERRY_PER_GROUP ? ilog2_exact(p.gw) : 0;
    p.spr = s.granularity == SHERRY_PER_GROUP ? (int)(s.K / s.group) : 0;
    if (!vec4)
        p.mode = kModeGen;
    else if (p.row_scale)
        p.mode = kModeRow;
    else if (p.gw_shift >= 2)
        p.mode = kModeStep;
    else if (p.gw_shift >= 0)
        p.mode = kModeWord;
    else
        p.mode = kModeGen;
}

// Tile plan: R = 32*WR rows per CTA tile; K split S ways so that a launch has
// enough tiles to fill the GPU (about two CTAs per SM).
static Plan make_plan(const ProbShape* shapes, int count, int64_t M, int sms) {
    Plan pl;
    pl.MT = tokens_per_pass(M);
    const int n_pass = (int)((M + pl.MT - 1) / pl.MT);
    const int target = 2 * sms;
    int64_t rows_total = 0;
    for (int i = 0; i < count; ++i) rows_total += shapes[i].N;
    // fewer rows -> smaller row tiles
    pl.WR = (rows_total * n_pass >= (int64_t)256 * target) ? 8 : 2;
    const int R = 32 * pl.WR;
    int64_t tiles_nosplit = 0;
    for (int i = 0; i < count; ++i) tiles_nosplit += n_pass * ((shapes[i].N + R - 1) / R);
    size_t cnt_ints = 0, part_floats = 0;
    int tb = 0;
    const int ksw = (kLutTables / pl.MT) / 8;  // words per sub-slice
    for (int i = 0; i < count; ++i) {
        const ProbShape& s = shapes[i];
        LinProb p{};
        fill_mode(p, s);
        p.N = (int)s.N;
        p.K = (int)s.K;
        p.n_rt = (int)((s.N + R - 1) / R);
        p.n_pass = n_pass;
        const int words = (int)(s.K / 32);
        int S = 1;
        if (tiles_nosplit < target) {
            // split K so this problem's tiles reach its share of the target
            const int64_t mine = (int64_t)n_pass * p.n_rt;
            const int64_t want = std::max<int64_t>(1, (int64_t)target * mine / std::max<int64_t>(1, tiles_nosplit));
            S = (int)std::min<int64_t>((want + mine - 1) / mine, std::max(1, words / 4));
        }
        // words per split: whole sub-slices when possible, else whole 4-word steps
        int wps = (words + S - 1) / S;
        const int gran = (wps >= ksw) ? ksw : 4;
        wps = ((wps + gran - 1) / gran) * gran;
        if (p.mode == kModeGen) wps = (words + S - 1) / S;  // any word count
        S = (words + wps - 1) / wps;
        p.S = S;
        p.wps = wps;
        p.tile_begin = tb;
        tb += n_pass * p.n_rt * S;
        if (S > 1) {
            cnt_ints += (size_t)n_pass * p.n_rt;
            part_floats += (size_t)n_pass * p.n_rt * S * pl.MT * R;
        }
        pl.probs.push_back(p);
    }
    pl.total_tiles = tb;
    const size_t cnt_bytes = kTicketBytes;
    pl.ws_bytes = cnt_ints ? cnt_bytes + part_floats * sizeof(float) : 0;
    // assign workspace slices
    size_t ci = 0, pf = 0;
    for (auto& p : pl.probs) {
        if (p.S > 1) {
            p.cnt = reinterpret_cast<int*>((uintptr_t)ci * sizeof(int));  // offsets, rebased at launch
            p.part = reinterpret_cast<float*>(cnt_bytes + pf * sizeof(float));
            ci += (size_t)p.n_pass * p.n_rt;
            pf += (size_t)p.n_pass * p.n_rt * p.S * pl.MT * 32 * pl.WR;
        }
    }
    return pl;
}

size_t lut_workspace_bytes(const ProbShape* shapes, int count, int64_t M, int sms) {
    return make_plan(shapes, count, M, sms).ws_bytes;
}

template <int MT, int WR, int MAXP>
static int launch_plan_t(const Plan& pl, int64_t M, int y_bf16, int sms, cudaStream_t stream) {
    static LinParams<MAXP> P;  // large: keep off the stack
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    P.count = (int)pl.probs.size();
    P.M = (int)M;
    P.y_bf16 = y_bf16;
    P.total_tiles = pl.total_tiles;
    for (int i = 0; i < P.count; ++i) P.p[i] = pl.probs[i];
    auto kern = k_lut_linear<MT, WR, MAXP>;
    static PerDevice occ_dev;
    int occ = 0;
    const int st = per_device(occ_dev, &occ, [&](int& v) {
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutSmem));
        SHERRY_CUDA_CHECK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, kLThreads, kLutSmem));
        if (v < 1) v = 1;
        return SHERRY_OK;
    });
    if (st) return st;
    const int grid = std::min(pl.total_tiles, occ * sms);
    kern<<<grid, kLThreads, kLutSmem, stream>>>(P);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

template <int MT, int WR>
static int launch_plan_p(const Plan& pl, int64_t M, int y_bf16, int sms, cudaStream_t stream) {
    const size_t c = pl.probs.size();
    if (c <= 1) return launch_plan_t<MT, WR, 1>(pl, M, y_bf16, sms, stream);
    if (c <= 16) return launch_plan_t<MT, WR, 16>(pl, M, y_bf16, sms, stream);
    return launch_plan_t<MT, WR, SHERRY_MAX_BATCH>(pl, M, y_bf16, sms, stream);
}

// descs: X, idx, sgn, scales, Y of each problem
int lut_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M,
                      int y_bf16, void* workspace, int sms, cudaStream_t stream) {
    Plan pl = make_plan(shapes, count, M, sms);
    for (int i = 0; i < count; ++i) {
        LinProb& p = pl.probs[i];
        p.X = descs[i].X;
        p.idx = descs[i].idx;
        p.sgn = descs[i].sgn;
        p.scales = descs[i].scales;
        p.Y = descs[i].Y;
        if (p.S > 1) {
            char* ws = static_cast<char*>(workspace);
            p.cnt = reinterpret_cast<int*>(ws + reinterpret_cast<uintptr_t>(p.cnt));
            p.part = reinterpret_cast<float*>(ws + reinterpret_cast<uintptr_t>(p.part));
        } else {
            p.cnt = nullptr;
            p.part = nullptr;
        }
    }
    if (pl.total_tiles == 0) return SHERRY_OK;
    const int mt = pl.MT, wr = pl.WR;
    if (mt == 1) return wr == 8 ? launch_plan_p<1, 8>(pl, M, y_bf16, sms, stream)
                                : launch_plan_p<1, 2>(pl, M, y_bf16, sms, stream);
    if (mt == 2) return wr == 8 ? launch_plan_p<2, 8>(pl, M, y_bf16, sms, stream)
                                : launch_plan_p<2, 2>(pl, M, y_bf16, sms, stream);
    return wr == 8 ? launch_plan_p<4, 8>(pl, M, y_bf16, sms, stream)
                   : launch_plan_p<4, 2>(pl, M, y_bf16, sms, stream);
}

}  // namespace sherry
