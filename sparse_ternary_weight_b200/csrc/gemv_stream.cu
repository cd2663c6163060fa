// gemv_stream.cu -- packed 3:4 ternary linear, one token (M = 1), HBM-streaming
// version of the lookup-table decode (the method's inference scheme: tables
// built from the activations, looked up by the packed weights, accumulated,
// then scaled; "Sherry: Hardware-Efficient 1.25-Bit Ternary Quantization via
// Fine-grained Sparsification", digest paragraph on inference; Y = X T alpha).
//
// Work unit: 256 output rows x 1024 weights (32 packed words) of one linear.
// All units of a launch (one or many independent linears) are split into equal
// contiguous ranges, one per CTA (stream-K): every CTA streams the same number
// of bytes.  A row block whose units straddle two CTAs is finished by the CTA
// that arrives last at its ticket, adding the partial sums in unit order, so Y
// is deterministic.
//
// Per unit the CTA copies the packed planes with 16-byte cp.async (each 8
// threads read one full 128-byte row segment, so global reads are coalesced)
// into an XOR-swizzled shared layout that the row-per-lane reads hit without
// bank conflicts; three stages are in flight.  The 32-entry tables of the
// unit's 256 blocks of activations are double buffered and built one unit
// ahead.  A lane owns one row: per packed word it spreads the 8 nibbles and
// sign bits into two byte-vectors of table offsets (see lut.cuh) and does 8
// lookups; alpha is applied once per 128-weight group (or once per row).
#include "common.cuh"
#include "lut.cuh"

#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <vector>

namespace sherry {

constexpr int kSThreads = 512;                     // 16 warps: 8 row-warps x 2 K-halves
constexpr int kSRows = 256;                        // rows per unit, one per lane of a row-warp
constexpr int kSWords = 32;                        // packed words per unit
constexpr int kSStages = 3;
constexpr int kSIdx = kSRows * kSWords * 4;        // 32 KB
constexpr int kSSgn = kSRows * kSWords;            // 8 KB
constexpr int kSSc = kSRows * 32;                  // 8 KB (at most 8 fp32 scales per row)
constexpr int kSStage = kSIdx + kSSgn + kSSc;      // 48 KB
constexpr int kSLut = 256 * kTab;                  // 36 KB, one table per block of the unit
constexpr int kSSmem = kSStages * kSStage + 2 * kSLut + 256;
static_assert(kSStage % 256 == 0 && kSLut % 256 == 0, "table bases must stay multiples of 256");

enum SMode { kSRow = 0, kSG128 = 1, kSG256 = 2 };

struct SProb {
    const uint16_t* X;
    const uint32_t* idx;
    const uint8_t* sgn;
    const float* scales;
    void* Y;
    int N, words, spr;  // spr: scales per row (per-group)
    int mode, per_tensor;
    int n_rb, n_sub;    // row blocks, sub-slices (units) per row block
    int unit_begin, tile_begin;
};

template <int MAXP>
struct SParams {
    int count, y_bf16, total_units, upc;
    float* part;  // [grid][2][kSRows] split-tile partials
    int* ticket;  // [total tiles]
    SProb p[MAXP];
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

extern __shared__ __align__(16) unsigned char g_smem[];

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// 8 lookups of one packed word (tables of blocks BOFF..BOFF+7 at shared address
// `base`, a multiple of 256) -> even-position and odd-position partial sums
template <int BOFF>
__device__ __forceinline__ void word_sums(uint32_t w, uint32_t s, uint32_t base, float& p0, float& p1) {
    uint32_t ev, od;
    spread_word(w, s, ev, od);
    const float v0 = lds_imm<(BOFF + 0) * kTab>(__byte_perm(ev, base, 0x7650u));
    const float v1 = lds_imm<(BOFF + 1) * kTab>(__byte_perm(od, base, 0x7650u));
    const float v2 = lds_imm<(BOFF + 2) * kTab>(__byte_perm(ev, base, 0x7651u));
    const float v3 = lds_imm<(BOFF + 3) * kTab>(__byte_perm(od, base, 0x7651u));
    const float v4 = lds_imm<(BOFF + 4) * kTab>(__byte_perm(ev, base, 0x7652u));
    const float v5 = lds_imm<(BOFF + 5) * kTab>(__byte_perm(od, base, 0x7652u));
    const float v6 = lds_imm<(BOFF + 6) * kTab>(__byte_perm(ev, base, 0x7653u));
    const float v7 = lds_imm<(BOFF + 7) * kTab>(__byte_perm(od, base, 0x7653u));
    p0 = (v0 + v2) + (v4 + v6);
    p1 = (v1 + v3) + (v5 + v7);
}

struct UnitPos {
    int p, rb, sub;  // problem, row block, sub-slice
};

// issue the cp.async copies of one unit into `stage`
template <int MAXP>
__device__ __forceinline__ void issue_unit(const SParams<MAXP>& P, const UnitPos& u, uint32_t stage) {
    const SProb& pr = P.p[u.p];
    const int t = threadIdx.x;
    const int row0 = u.rb * kSRows;
    const int w0 = u.sub * kSWords;
    const int words = pr.words, N = pr.N;
    {
        const int r0 = t >> 3, c = t & 7;
        const int word = w0 + 4 * c;
        const bool wok = word < words;
        const uint32_t* src = pr.idx + (int64_t)(row0 + r0) * words + word;
        const int64_t stepw = (int64_t)64 * words;
        uint32_t dst = stage + r0 * 128 + ((c ^ (r0 & 7)) << 4);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool ok = wok && (row0 + r0 + 64 * i) < N;
            cp_async16(dst + i * 64 * 128, ok ? src + i * stepw : pr.idx, ok);
        }
    }
    {
        const int r = t >> 1, h = t & 1;
        const int row = row0 + r, off = w0 + 16 * h;
        const bool ok = row < N && off < words;
        cp_async16(stage + kSIdx + r * 32 + ((h ^ ((r >> 2) & 1)) << 4), ok ? pr.sgn + (int64_t)row * words + off : pr.sgn, ok);
        if (pr.mode == kSG128) {
            const int offs = w0 / 4 + 4 * h;
            const bool oks = row < N && offs < pr.spr;
            cp_async16(stage + kSIdx + kSSgn + r * 32 + ((h ^ ((r >> 2) & 1)) << 4),
                       oks ? pr.scales + (int64_t)row * pr.spr + offs : pr.scales, oks);
        }
    }
    if (pr.mode == kSG256 && t < kSRows) {
        const int r = t;
        const int row = row0 + r, off = w0 / 8;
        const bool ok = row < N && off < pr.spr;
        cp_async16(stage + kSIdx + kSSgn + r * 32 + (((r >> 2) & 1) << 4), ok ? pr.scales + (int64_t)row * pr.spr + off : pr.scales, ok);
    }
}

template <int MAXP>
__device__ __forceinline__ UnitPos locate(const SParams<MAXP>& P, int u) {
    int p = 0;
    while (p + 1 < P.count && P.p[p + 1].unit_begin <= u) ++p;
    const int local = u - P.p[p].unit_begin;
    return UnitPos{p, local / P.p[p].n_sub, local % P.p[p].n_sub};
}

__device__ __forceinline__ void advance(const SProb* probs, UnitPos& u) {
    if (++u.sub == probs[u.p].n_sub) {
        u.sub = 0;
        if (++u.rb == probs[u.p].n_rb) {
            u.rb = 0;
            ++u.p;
        }
    }
}

// Half of the 32-entry table of one block of 4 activations: the entries with
// zero position z in {2h, 2h+1} and their negations.
__device__ __forceinline__ void build_half_table(uint32_t tab, uint2 xb, int h) {
    const float x0 = bf16lo(xb.x), x1 = bf16hi(xb.x), x2 = bf16lo(xb.y), x3 = bf16hi(xb.y);
    // z = 2h: kept (h ? x0,x1,x3 : x1,x2,x3); z = 2h+1: kept (h ? x0,x1,x2 : x0,x2,x3)
    const float a0 = h ? x0 : x1, b0 = h ? x1 : x2, c0 = x3;
    const float a1 = x0, b1 = h ? x1 : x2, c1 = h ? x2 : x3;
    const float s0 = a0 + b0, d0 = a0 - b0, s1 = a1 + b1, d1 = a1 - b1;
    const float e0 = s0 + c0, e1 = s0 - c0, e2 = d0 + c0, e3 = d0 - c0;
    const float e4 = s1 + c1, e5 = s1 - c1, e6 = d1 + c1, e7 = d1 - c1;
    const uint32_t o = tab + 32 * h;
    sts_v4(o, e0, e1, e2, e3);
    sts_v4(o + 16, e4, e5, e6, e7);
    sts_v4(o + 64, -e0, -e1, -e2, -e3);
    sts_v4(o + 80, -e4, -e5, -e6, -e7);
}

// Lookups of one row over steps [4*kh, 4*kh + nst) of a unit (4 words each);
// `st` and `lut` are byte offsets into the dynamic shared buffer.
template <int MODE, bool FULL>
__device__ __forceinline__ float unit_rows(uint32_t st, uint32_t lut, int r, int kh, int nst) {
    const uint32_t sw2 = ((r >> 2) & 1) << 4;
    const uint4 sg = lds128(st + kSIdx + r * 32 + ((uint32_t)(kh << 4) ^ sw2));
    uint4 av = make_uint4(0u, 0u, 0u, 0u);
    if (MODE == kSG128) av = lds128(st + kSIdx + kSSgn + r * 32 + ((uint32_t)(kh << 4) ^ sw2));
    if (MODE == kSG256) av = lds128(st + kSIdx + kSSgn + r * 32 + sw2);
    const uint32_t idx_row = st + r * 128;
    const uint32_t sw8 = (uint32_t)(r & 7);
    float acc = 0.0f;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        if (FULL || cc < nst) {
            const int c = 4 * kh + cc;
            const uint4 wq = lds128(idx_row + (((uint32_t)c ^ sw8) << 4));
            const uint32_t sq = cc == 0 ? sg.x : cc == 1 ? sg.y : cc == 2 ? sg.z : sg.w;
            const uint32_t tb = lut + (uint32_t)(c * 32 * kTab);
            float p0, p1, q0, q1, r0, r1, u0, u1;
            word_sums<0>(wq.x, sq & 0xffu, tb, p0, p1);
            word_sums<8>(wq.y, (sq >> 8) & 0xffu, tb, q0, q1);
            word_sums<16>(wq.z, (sq >> 16) & 0xffu, tb, r0, r1);
            word_sums<24>(wq.w, sq >> 24, tb, u0, u1);
            const float s4 = ((p0 + q0) + (r0 + u0)) + ((p1 + q1) + (r1 + u1));
            if (MODE == kSRow) {
                acc += s4;
            } else {
                uint32_t ab;
                if (MODE == kSG128)
                    ab = cc == 0 ? av.x : cc == 1 ? av.y : cc == 2 ? av.z : av.w;
                else {
                    const int gi = c >> 1;
                    ab = gi == 0 ? av.x : gi == 1 ? av.y : gi == 2 ? av.z : av.w;
                }
                acc = fmaf(__uint_as_float(ab), s4, acc);
            }
        }
    }
    return acc;
}

template <int MODE>
__device__ __forceinline__ float unit_rows_any(uint32_t st, uint32_t lut, int r, int kh, int nst) {
    return nst == 4 ? unit_rows<MODE, true>(st, lut, r, kh, 4) : unit_rows<MODE, false>(st, lut, r, kh, nst);
}

template <int MAXP>
__global__ void __launch_bounds__(kSThreads, 1) k_lut_stream(const __grid_constant__ SParams<MAXP> P) {
    __shared__ int s_last;
    __shared__ float s_half[kSRows];
    // Shared addresses: the buffer is rounded up to 256 bytes, so every table
    // base is a multiple of 256 (a lookup's address replaces its low byte); the
    // XOR swizzles need only 16-byte alignment, since writer and reader apply them.
    const uint32_t stages = (smem_u32(g_smem) + 255u) & ~255u;
    const uint32_t luts = stages + kSStages * kSStage;

    const int t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    const int r = (warp & 7) * 32 + lane;  // row within the unit
    const int kh = warp >> 3;              // K half of the unit: steps 4kh .. 4kh+3
    const int tb_idx = t & 255, tb_half = t >> 8;  // table-building role
    const int u_begin = blockIdx.x * P.upc;
    const int u_end = min(P.total_units, u_begin + P.upc);
    if (u_begin >= u_end) return;

    // prologue: units u_begin .. u_begin + kSStages - 2 in flight
    UnitPos pre = locate(P, u_begin);
    for (int i = 0; i < kSStages - 1; ++i) {
        if (u_begin + i < u_end) {
            issue_unit(P, pre, stages + i * kSStage);
            advance(P.p, pre);
        }
        cp_async_commit();
    }
    UnitPos cur = locate(P, u_begin);
    {
        const SProb& pr = P.p[cur.p];
        const int b = cur.sub * kSWords * 8 + tb_idx;
        if (b < pr.words * 8)
            build_half_table(luts + tb_idx * kTab, __ldg(reinterpret_cast<const uint2*>(pr.X) + b), tb_half);
    }
    bool tile_from_start = (P.p[cur.p].unit_begin + cur.rb * P.p[cur.p].n_sub == u_begin);
    float acc = 0.0f;

    for (int u = u_begin; u < u_end; ++u) {
        const int k = u - u_begin;
        cp_async_wait<kSStages - 2>();
        __syncthreads();
        if (u + kSStages - 1 < u_end)
            issue_unit(P, pre, stages + ((k + kSStages - 1) % kSStages) * kSStage);
        cp_async_commit();
        if (u + kSStages - 1 < u_end) advance(P.p, pre);

        // activations of the next unit's tables (latency hidden by this unit)
        UnitPos nxt = cur;
        advance(P.p, nxt);
        uint2 xn = make_uint2(0u, 0u);
        bool xn_ok = false;
        if (u + 1 < u_end) {
            const SProb& pn = P.p[nxt.p];
            const int b = nxt.sub * kSWords * 8 + tb_idx;
            xn_ok = b < pn.words * 8;
            if (xn_ok) xn = __ldg(reinterpret_cast<const uint2*>(pn.X) + b);
        }

        const SProb& pr = P.p[cur.p];
        const uint32_t st = stages + (k % kSStages) * kSStage;
        const uint32_t lut = luts + (k & 1) * kSLut;
        const int nst = min(4, ((pr.words - cur.sub * kSWords) >> 2) - 4 * kh);
        if (nst > 0) {
            if (pr.mode == kSRow)
                acc += unit_rows_any<kSRow>(st, lut, r, kh, nst);
            else if (pr.mode == kSG128)
                acc += unit_rows_any<kSG128>(st, lut, r, kh, nst);
            else
                acc += unit_rows_any<kSG256>(st, lut, r, kh, nst);
        }

        const bool tile_end = (cur.sub == pr.n_sub - 1);
        if (tile_end || u == u_end - 1) {
            // the two K halves of each row, in a fixed order
            if (kh == 1) s_half[r] = acc;
            __syncthreads();
            const int n = cur.rb * kSRows + r;
            const bool row_ok = n < pr.N;
            float v = acc + s_half[r];
            if (pr.mode == kSRow && row_ok) v *= __ldg(pr.scales + (pr.per_tensor ? 0 : n));
            if (tile_from_start && tile_end) {
                if (kh == 0 && row_ok) {
                    if (P.y_bf16)
                        reinterpret_cast<__nv_bfloat16*>(pr.Y)[n] = __float2bfloat16_rn(v);
                    else
                        reinterpret_cast<float*>(pr.Y)[n] = v;
                }
            } else {
                // split tile: partial into this CTA's slot, then the ticket
                const int tile = pr.tile_begin + cur.rb;
                const int tile_u0 = pr.unit_begin + cur.rb * pr.n_sub;
                const int c_a = tile_u0 / P.upc;
                const int c_b = (tile_u0 + pr.n_sub - 1) / P.upc;
                const int slot = (u_begin >= tile_u0) ? 0 : 1;
                if (kh == 0) __stcg(P.part + ((int64_t)blockIdx.x * 2 + slot) * kSRows + r, v);
                __threadfence();
                __syncthreads();
                if (t == 0) s_last = (atomicAdd(P.ticket + tile, 1) == c_b - c_a);
                __syncthreads();
                if (s_last && kh == 0) {
                    __threadfence();
                    float sum = 0.0f;
                    for (int c = c_a; c <= c_b; ++c) {
                        const int sl = (c * P.upc >= tile_u0) ? 0 : 1;
                        const float pv = __ldcg(P.part + ((int64_t)c * 2 + sl) * kSRows + r);
                        sum = (c == c_a) ? pv : sum + pv;
                    }
                    if (row_ok) {
                        if (P.y_bf16)
                            reinterpret_cast<__nv_bfloat16*>(pr.Y)[n] = __float2bfloat16_rn(sum);
                        else
                            reinterpret_cast<float*>(pr.Y)[n] = sum;
                    }
                    if (t == 0) P.ticket[tile] = 0;  // leave the ticket zeroed
                }
            }
            acc = 0.0f;
            tile_from_start = true;  // every later tile of this range starts inside it
        }

        // tables of the next unit into the other buffer (its last reader was unit u-1)
        if (u + 1 < u_end && xn_ok) build_half_table(luts + ((k + 1) & 1) * kSLut + tb_idx * kTab, xn, tb_half);
        cur = nxt;
    }
    cp_async_wait<0>();
}

// ---- host side -------------------------------------------------------------------

bool stream_eligible(const ProbShape& s, int64_t M) {
    if (M != 1 || s.N == 0) return false;
    if ((s.N + kSRows - 1) / kSRows > kMaxTickets) return false;
    if (s.K % 512 != 0) return false;
    if (s.granularity == SHERRY_PER_TENSOR || s.granularity == SHERRY_PER_CHANNEL) return true;
    if (s.granularity != SHERRY_PER_GROUP) return false;
    if (s.group == 128) return true;                        // K/128 % 4 == 0 since K % 512 == 0
    if (s.group == 256) return (s.K / 256) % 4 == 0;        // 16-byte aligned scale rows
    return false;
}

struct SPlan {
    std::vector<SProb> probs;
    int total_units = 0, total_tiles = 0, grid = 0, upc = 0;
    size_t ws_bytes = 0, part_off = 0;
};

static int stream_ctas(int sms) { return sms; }  // one CTA per SM (the stages fill shared memory)

static SPlan make_splan(const ProbShape* shapes, int count, int sms) {
    SPlan pl;
    int ub = 0, tb = 0;
    for (int i = 0; i < count; ++i) {
        const ProbShape& s = shapes[i];
        SProb p{};
        p.N = (int)s.N;
        p.words = (int)(s.K / 32);
        p.spr = s.granularity == SHERRY_PER_GROUP ? (int)(s.K / s.group) : 0;
        p.mode = s.granularity != SHERRY_PER_GROUP ? kSRow : (s.group == 128 ? kSG128 : kSG256);
        p.per_tensor = s.granularity == SHERRY_PER_TENSOR;
        p.n_rb = (int)((s.N + kSRows - 1) / kSRows);
        p.n_sub = (p.words + kSWords - 1) / kSWords;
        p.unit_begin = ub;
        p.tile_begin = tb;
        ub += p.n_rb * p.n_sub;
        tb += p.n_rb;
        pl.probs.push_back(p);
    }
    pl.total_units = ub;
    pl.total_tiles = tb;
    const int g = std::max(1, std::min(stream_ctas(sms), ub));
    pl.upc = (ub + g - 1) / g;
    pl.grid = (ub + pl.upc - 1) / pl.upc;
    pl.part_off = kTicketBytes;
    pl.ws_bytes = kTicketBytes + (size_t)pl.grid * 2 * kSRows * sizeof(float);
    return pl;
}

size_t stream_workspace_bytes(const ProbShape* shapes, int count, int sms) {
    return make_splan(shapes, count, sms).ws_bytes;
}

template <int MAXP>
static int stream_launch_t(SPlan& pl, int y_bf16, void* workspace, cudaStream_t stream) {
    static SParams<MAXP> P;
    static std::mutex mu;
    static bool attr = false;
    std::lock_guard<std::mutex> lk(mu);
    P.count = (int)pl.probs.size();
    P.y_bf16 = y_bf16;
    P.total_units = pl.total_units;
    P.upc = pl.upc;
    P.ticket = static_cast<int*>(workspace);
    P.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.part_off);
    for (int i = 0; i < P.count; ++i) P.p[i] = pl.probs[i];
    if (!attr) {
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_lut_stream<MAXP>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSSmem));
        attr = true;
    }
    k_lut_stream<MAXP><<<pl.grid, kSThreads, kSSmem, stream>>>(P);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

int stream_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int y_bf16,
                         void* workspace, int sms, cudaStream_t stream) {
    SPlan pl = make_splan(shapes, count, sms);
    for (int i = 0; i < count; ++i) {
        SProb& p = pl.probs[i];
        p.X = descs[i].X;
        p.idx = descs[i].idx;
        p.sgn = descs[i].sgn;
        p.scales = descs[i].scales;
        p.Y = descs[i].Y;
    }
    if (pl.total_units == 0) return SHERRY_OK;
    if (count <= 1) return stream_launch_t<1>(pl, y_bf16, workspace, stream);
    if (count <= 16) return stream_launch_t<16>(pl, y_bf16, workspace, stream);
    return stream_launch_t<SHERRY_MAX_BATCH>(pl, y_bf16, workspace, stream);
}

}  // namespace sherry
