// gemv_stream.cu -- packed 3:4 ternary linear for one or two tokens (M <= 2),
// HBM-streaming version of the lookup-table decode (the method's inference
// scheme: tables built from the activations, looked up by the packed weights,
// accumulated, then scaled; "Sherry: Hardware-Efficient 1.25-Bit Ternary
// Quantization via Fine-grained Sparsification", digest paragraph on inference;
// Y = X T alpha).
//
// Work unit: 512 output rows x 512 weights (16 packed words) of one linear.
// All units of a launch (one or many independent linears) are split into equal
// contiguous ranges, one per CTA (stream-K): every CTA streams the same number
// of bytes.  A row block whose units straddle two CTAs is finished by the CTA
// that arrives last at its ticket, adding the partial sums in CTA order, so Y
// is deterministic.
//
// Roles (20 warps).  16 consumer warps: each thread owns one row of the unit
// and only looks up and accumulates (per packed word it spreads the 8 nibbles
// and sign bits into two byte-vectors of table offsets, see lut.cuh, and does 8
// lookups per token at the same offsets; alpha is applied once per 128-weight
// group, or once per row).  4 helper warps, one per SM sub-partition: they copy
// each unit's packed planes with 16-byte cp.async (4 lanes read one row's 64
// contiguous bytes, so global reads are coalesced) into an XOR-swizzled ring of
// stages (three for one token, two for two) that the row-per-lane reads hit
// without bank conflicts, and build the unit's 128 tables of 32 entries per
// token into the stage's table buffer.  Stages change hands through mbarriers;
// every wait is bounded, and a timeout sets a device status flag (reported by
// sherry_device_status) and ends the CTA.
#include "common.cuh"
#include "lut.cuh"

#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

namespace sherry {

constexpr int kSConsumers = 16;                    // consumer warps: one row per thread
constexpr int kSHelpers = 4;                       // copy + table warps
constexpr int kSThreads = 32 * (kSConsumers + kSHelpers);
constexpr int kSRows = 32 * kSConsumers;           // 512 rows per unit
constexpr int kSWords = 16;                        // packed words per unit (512 weights)
constexpr int kSIdx = kSRows * kSWords * 4;        // 32 KB
constexpr int kSSgn = kSRows * 16;                 // 8 KB (16 sign bytes per row)
constexpr int kSSc = kSRows * 16;                  // 8 KB (at most 4 fp32 scales per row)
constexpr int kSStage = kSIdx + kSSgn + kSSc;      // 48 KB
constexpr int kSTabs = kSWords * 8;                // 128 tables per unit
constexpr int kSLut = kSTabs * kTab;               // 18 KB: one token's tables of a unit
constexpr int kSBars = 128;                        // mbarriers
static_assert(kSStage % 256 == 0 && kSLut % 256 == 0, "table bases must stay multiples of 256");

// Ring depth and shared bytes for MT tokens (tables are token-major within a stage).
template <int MT>
struct SCfg {
    static constexpr int kStages = MT == 1 ? 3 : 2;
    static constexpr int kLutStage = MT * kSLut;
    static constexpr int kSmem = 256 + kStages * (kSStage + kLutStage) + kSBars;
};
static_assert(SCfg<1>::kSmem <= 232448 && SCfg<2>::kSmem <= 232448, "shared memory per CTA");
static_assert(kSTabs == 32 * kSHelpers, "one table per helper thread");
constexpr long long kSWaitCycles = 4000000000LL;   // default wait budget, ~2 s at the boost clock
// The no-workspace entry point's fixed scratch holds this kernel's largest plan
// (two tokens, one CTA per SM, two partial slots per CTA) on up to 224 SMs.
static_assert(kTicketBytes + (size_t)224 * 2 * 2 * kSRows * sizeof(float) <= SHERRY_NOALLOC_SCRATCH_BYTES,
              "no-workspace scratch too small for the streaming plan");

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
    long long wait_cycles;  // budget of every bounded wait, in SM clock cycles
    int count, y_bf16, total_units, upc;
    float* part;  // [grid][2][MT][kSRows] split-tile partials
    int* ticket;  // [total tiles]
    SProb p[MAXP];
};

// bounded-wait timeouts of this file's kernel (read and cleared by sherry_device_status)
__device__ int g_stream_status = 0;

namespace {

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(valid ? 8 : 0)
                 : "memory");
}
// the mbarrier receives one arrival when all of this thread's prior cp.async complete
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// wait for the phase with the given parity to complete; false on timeout (after
// `budget` cycles) or when another thread of the CTA has given up
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, long long budget) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > budget) {
            *abort_flag = 1;
            atomicExch(&g_stream_status, SHERRY_ERR_TIMEOUT);
            return false;
        }
    }
}

}  // namespace

extern __shared__ __align__(16) unsigned char g_smem[];

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

// 8 lookups of one packed word for token TOK: the tables of blocks BOFF..BOFF+7
// sit at shared offsets (BOFF + j) * kTab + TOK * kSLut from the addresses in a[],
// whose low byte is the block's table offset -> even-position and odd-position
// partial sums p0 = (v0 + v2) + (v4 + v6), p1 = (v1 + v3) + (v5 + v7), as
// packed pair adds
template <int BOFF, int TOK>
__device__ __forceinline__ void token_sums(const uint32_t (&a)[8], float& p0, float& p1) {
    constexpr int T = TOK * kSLut;
    const float v0 = lds_imm<(BOFF + 0) * kTab + T>(a[0]);
    const float v1 = lds_imm<(BOFF + 1) * kTab + T>(a[1]);
    const float v2 = lds_imm<(BOFF + 2) * kTab + T>(a[2]);
    const float v3 = lds_imm<(BOFF + 3) * kTab + T>(a[3]);
    const float v4 = lds_imm<(BOFF + 4) * kTab + T>(a[4]);
    const float v5 = lds_imm<(BOFF + 5) * kTab + T>(a[5]);
    const float v6 = lds_imm<(BOFF + 6) * kTab + T>(a[6]);
    const float v7 = lds_imm<(BOFF + 7) * kTab + T>(a[7]);
    float a0, a1, b0, b1;
    add2(a0, a1, v0, v1, v2, v3);
    add2(b0, b1, v4, v5, v6, v7);
    add2(p0, p1, a0, a1, b0, b1);
}

// One packed word (nibbles w, sign byte s; its 8 tables at `base`, a multiple of
// 256, plus BOFF * kTab): the 8 table addresses are formed once and looked up for
// each of the MT tokens.
template <int BOFF, int MT>
__device__ __forceinline__ void word_sums(uint32_t w, uint32_t s, uint32_t base, float (&p0)[MT], float (&p1)[MT]) {
    uint32_t ev, od;
    spread_word(w, s, ev, od);
    const uint32_t a[8] = {__byte_perm(ev, base, 0x7650u), __byte_perm(od, base, 0x7650u),
                           __byte_perm(ev, base, 0x7651u), __byte_perm(od, base, 0x7651u),
                           __byte_perm(ev, base, 0x7652u), __byte_perm(od, base, 0x7652u),
                           __byte_perm(ev, base, 0x7653u), __byte_perm(od, base, 0x7653u)};
    token_sums<BOFF, 0>(a, p0[0], p1[0]);
    if constexpr (MT > 1) token_sums<BOFF, 1>(a, p0[1], p1[1]);
}

struct UnitPos {
    int p, rb, sub;  // problem, row block, sub-slice
};

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

// Copy geometry of helper lane (h, lane) for one row block: the unit's rows
// [128h, 128h+128).  Packed words: rows 128h + 8i + lane/4 (i = 0..15), 16-byte
// chunk lane%4 of the row's 64 bytes, stored at chunk (c ^ ((row >> 1) & 3)) of a
// 64-byte shared row (that swizzle term is (lane >> 3) & 3 for every i).  Sign
// bytes and scales: rows 128h + 32i + lane (i = 0..3), 16 bytes each.  Byte
// offsets from the plane bases; a row past N reads row 0 instead (its results
// are never stored), so every copy is a full in-bounds 16 bytes.
struct CopyRows {
    uint32_t idx[16], sgn[4], sc[4];
};

__device__ __forceinline__ void copy_rows(const SProb& pr, int rb, int h, int lane, CopyRows& cr) {
    const int row0 = rb * kSRows;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int row = row0 + 128 * h + 8 * i + (lane >> 2);
        cr.idx[i] = (uint32_t)((int64_t)(row < pr.N ? row : 0) * pr.words * 4 + 16 * (lane & 3));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = row0 + 128 * h + 32 * i + lane;
        const int rr = row < pr.N ? row : 0;
        cr.sgn[i] = (uint32_t)((int64_t)rr * pr.words);
        cr.sc[i] = (uint32_t)((int64_t)rr * pr.spr * 4);
    }
}

__device__ __forceinline__ const void* byte_off(const void* base, uint32_t off) {
    return static_cast<const char*>(base) + off;
}

// Helper lane's copies of unit (cr's row block, sub-slice `sub`) into `stage`.
__device__ __forceinline__ void copy_unit(const SProb& pr, const CopyRows& cr, int sub, uint32_t stage, int h,
                                          int lane) {
    const char* bi = reinterpret_cast<const char*>(pr.idx) + sub * (kSWords * 4);
    const uint32_t di = stage + (uint32_t)(128 * h + (lane >> 2)) * 64u +
                        ((uint32_t)((lane & 3) ^ ((lane >> 3) & 3)) << 4);
#pragma unroll
    for (int i = 0; i < 16; ++i) cp_async16(di + 512u * i, byte_off(bi, cr.idx[i]), true);
    const char* bs = reinterpret_cast<const char*>(pr.sgn) + sub * kSWords;
    const uint32_t ds = stage + kSIdx + (uint32_t)(128 * h + lane) * 16u;
#pragma unroll
    for (int i = 0; i < 4; ++i) cp_async16(ds + 512u * i, byte_off(bs, cr.sgn[i]), true);
    if (pr.mode == kSG128) {
        const char* ba = reinterpret_cast<const char*>(pr.scales) + sub * 16;
#pragma unroll
        for (int i = 0; i < 4; ++i) cp_async16(ds + kSSgn + 512u * i, byte_off(ba, cr.sc[i]), true);
    } else if (pr.mode == kSG256) {
        const char* ba = reinterpret_cast<const char*>(pr.scales) + sub * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) cp_async8(ds + kSSgn + 512u * i, byte_off(ba, cr.sc[i]), true);
    }
}

// Lookups of one row over the 16 words of a unit for MT tokens, into u[]; `st`
// and `lut` are shared addresses of the unit's stage and of token 0's tables.
template <int MODE, int MT>
__device__ __forceinline__ void unit_row(uint32_t st, uint32_t lut, int r, float (&u)[MT]) {
    const uint32_t sw = (uint32_t)((r >> 1) & 3);
    const uint4 sg = lds128(st + kSIdx + r * 16);
    uint4 av = make_uint4(0u, 0u, 0u, 0u);
    if (MODE == kSG128) av = lds128(st + kSIdx + kSSgn + r * 16);
    if (MODE == kSG256) {
        const uint2 a2 = lds64(st + kSIdx + kSSgn + r * 16);
        av = make_uint4(a2.x, a2.y, 0u, 0u);
    }
    const uint32_t idx_row = st + r * 64;
#pragma unroll
    for (int m = 0; m < MT; ++m) u[m] = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 wq = lds128(idx_row + (((uint32_t)q ^ sw) << 4));
        const uint32_t sq = q == 0 ? sg.x : q == 1 ? sg.y : q == 2 ? sg.z : sg.w;
        const uint32_t tb = lut + (uint32_t)(q * 32 * kTab);  // tables of words 4q..4q+3 (256-aligned)
        float p0[MT], p1[MT], q0[MT], q1[MT], r0[MT], r1[MT], u0[MT], u1[MT];
        word_sums<0, MT>(wq.x, sq & 0xffu, tb, p0, p1);
        word_sums<8, MT>(wq.y, (sq >> 8) & 0xffu, tb, q0, q1);
        word_sums<16, MT>(wq.z, (sq >> 16) & 0xffu, tb, r0, r1);
        word_sums<24, MT>(wq.w, sq >> 24, tb, u0, u1);
        uint32_t ab = 0u;
        if (MODE == kSG128) ab = q == 0 ? av.x : q == 1 ? av.y : q == 2 ? av.z : av.w;
        if (MODE == kSG256) ab = q < 2 ? av.x : av.y;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float e0, e1, f0, f1, g0, g1;
            add2(e0, e1, p0[m], p1[m], q0[m], q1[m]);
            add2(f0, f1, r0[m], r1[m], u0[m], u1[m]);
            add2(g0, g1, e0, e1, f0, f1);
            const float s4 = g0 + g1;  // ((p0 + q0) + (r0 + u0)) + ((p1 + q1) + (r1 + u1))
            if (MODE == kSRow)
                u[m] += s4;
            else
                u[m] = fmaf(__uint_as_float(ab), s4, u[m]);
        }
    }
}

template <int MAXP, int MT>
__global__ void __launch_bounds__(kSThreads, 1) k_lut_stream(const __grid_constant__ SParams<MAXP> P) {
    using C = SCfg<MT>;
    constexpr int S = C::kStages;
    __shared__ int s_last;
    __shared__ int s_abort;
    // Shared addresses: the buffer is rounded up to 256 bytes, so every table
    // base is a multiple of 256 (a lookup's address replaces its low byte); the
    // XOR swizzles need only 16-byte alignment, since writer and reader apply them.
    const uint32_t stages = (smem_u32(g_smem) + 255u) & ~255u;
    const uint32_t luts = stages + S * kSStage;  // table buffer s (MT tokens' tables) belongs to stage s
    const uint32_t bars = luts + S * C::kLutStage;
    // ready(s): the stage's planes landed and its tables are built; empty(s): consumers are done with both
    auto ready = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bars + 32u + 8u * (uint32_t)s; };
    const uint32_t bar_part = bars + 64u;  // every consumer stored its split-tile partial
    const uint32_t bar_last = bars + 72u;  // the ticket's outcome is in s_last

    const int t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    const int u_begin = blockIdx.x * P.upc;
    const int u_end = min(P.total_units, u_begin + P.upc);
    if (u_begin >= u_end) return;
    const int nu = u_end - u_begin;
    if (t == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(ready(s), 2 * 32 * kSHelpers);  // one cp.async arrival and one table arrival per helper thread
            mbar_init(empty(s), kSRows);
        }
        mbar_init(bar_part, kSRows);
        mbar_init(bar_last, 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int* abort_flag = &s_abort;

    if (warp >= kSConsumers) {
        // ---- helpers: unit j's copies and tables go to stage j % S once the
        // consumers are done with unit j - S there
        const int h = warp - kSConsumers;
        const int ht = t - 32 * kSConsumers;  // table (block of 4 activations) of the unit
        UnitPos cu = locate(P, u_begin);
        CopyRows cr;
        copy_rows(P.p[cu.p], cu.rb, h, lane, cr);
        // activations: token m's row of X starts K bf16 (words * 8 groups of 4) after token m-1's
        uint2 xb[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m)
            xb[m] = __ldg(reinterpret_cast<const uint2*>(P.p[cu.p].X) + (int64_t)m * P.p[cu.p].words * 8 +
                          cu.sub * kSTabs + ht);
        for (int j = 0; j < nu; ++j) {
            const int s = j % S;
            if (j >= S && !mbar_wait(empty(s), (uint32_t)(((j / S) & 1) ^ 1), abort_flag, P.wait_cycles)) break;
            const SProb& pr = P.p[cu.p];
            copy_unit(pr, cr, cu.sub, stages + s * kSStage, h, lane);
            cp_async_arrive(ready(s));
#pragma unroll
            for (int m = 0; m < MT; ++m) build_table(luts + s * C::kLutStage + m * kSLut + ht * kTab, xb[m]);
            mbar_arrive(ready(s));
            const int p0 = cu.p, rb0 = cu.rb;
            advance(P.p, cu);
            if (j + 1 < nu) {
                const SProb& pn = P.p[cu.p];
                if (cu.p != p0 || cu.rb != rb0) copy_rows(pn, cu.rb, h, lane, cr);
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    xb[m] = __ldg(reinterpret_cast<const uint2*>(pn.X) + (int64_t)m * pn.words * 8 + cu.sub * kSTabs +
                                  ht);
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        return;
    }

    // ---- consumers: thread t owns row t of every unit
    const int r = t;
    UnitPos cur = locate(P, u_begin);
    bool tile_from_start = (P.p[cur.p].unit_begin + cur.rb * P.p[cur.p].n_sub == u_begin);
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    int events = 0;  // split tiles handled so far (phase of bar_part / bar_last)
    for (int k = 0; k < nu; ++k) {
        const int s = k % S;
        if (!mbar_wait(ready(s), (uint32_t)((k / S) & 1), abort_flag, P.wait_cycles)) break;
        const SProb& pr = P.p[cur.p];
        const uint32_t st = stages + s * kSStage;
        const uint32_t lut = luts + s * C::kLutStage;
        float u[MT];
        if (pr.mode == kSRow)
            unit_row<kSRow, MT>(st, lut, r, u);
        else if (pr.mode == kSG128)
            unit_row<kSG128, MT>(st, lut, r, u);
        else
            unit_row<kSG256, MT>(st, lut, r, u);
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] += u[m];
        mbar_arrive(empty(s));

        const bool tile_end = (cur.sub == pr.n_sub - 1);
        if (tile_end || k == nu - 1) {
            const int n = cur.rb * kSRows + r;
            const bool row_ok = n < pr.N;
            float v[MT];
            const float rs = (pr.mode == kSRow && row_ok) ? __ldg(pr.scales + (pr.per_tensor ? 0 : n)) : 1.0f;
#pragma unroll
            for (int m = 0; m < MT; ++m) v[m] = pr.mode == kSRow ? acc[m] * rs : acc[m];
            if (tile_from_start && tile_end) {
                if (row_ok) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (P.y_bf16)
                            reinterpret_cast<__nv_bfloat16*>(pr.Y)[(int64_t)m * pr.N + n] = __float2bfloat16_rn(v[m]);
                        else
                            reinterpret_cast<float*>(pr.Y)[(int64_t)m * pr.N + n] = v[m];
                    }
                }
            } else {
                // split tile: partials into this CTA's slot, then the ticket
                const int tile = pr.tile_begin + cur.rb;
                const int tile_u0 = pr.unit_begin + cur.rb * pr.n_sub;
                const int c_a = tile_u0 / P.upc;
                const int c_b = (tile_u0 + pr.n_sub - 1) / P.upc;
                const int slot = (u_begin >= tile_u0) ? 0 : 1;
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    __stcg(P.part + (((int64_t)blockIdx.x * 2 + slot) * MT + m) * kSRows + r, v[m]);
                __threadfence();
                mbar_arrive(bar_part);
                const uint32_t ph = (uint32_t)(events & 1);
                ++events;
                if (r == 0) {
                    if (!mbar_wait(bar_part, ph, abort_flag, P.wait_cycles)) break;
                    s_last = (atomicAdd(P.ticket + tile, 1) == c_b - c_a);
                    mbar_arrive(bar_last);
                }
                if (!mbar_wait(bar_last, ph, abort_flag, P.wait_cycles)) break;
                if (s_last) {
                    __threadfence();
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        float sum = 0.0f;
                        for (int c = c_a; c <= c_b; ++c) {
                            const int sl = (c * P.upc >= tile_u0) ? 0 : 1;
                            const float pv = __ldcg(P.part + (((int64_t)c * 2 + sl) * MT + m) * kSRows + r);
                            sum = (c == c_a) ? pv : sum + pv;
                        }
                        if (row_ok) {
                            if (P.y_bf16)
                                reinterpret_cast<__nv_bfloat16*>(pr.Y)[(int64_t)m * pr.N + n] = __float2bfloat16_rn(sum);
                            else
                                reinterpret_cast<float*>(pr.Y)[(int64_t)m * pr.N + n] = sum;
                        }
                    }
                    if (r == 0) P.ticket[tile] = 0;  // leave the ticket zeroed
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
            tile_from_start = true;  // every later tile of this range starts inside it
        }
        advance(P.p, cur);
    }
}

// ---- host side -------------------------------------------------------------------

bool stream_eligible(const ProbShape& s, int64_t M) {
    if ((M != 1 && M != 2) || s.N == 0) return false;
    if ((s.N + kSRows - 1) / kSRows > kMaxTickets) return false;
    if (s.K % 512 != 0) return false;
    if (s.N * (s.K / 8) >= (int64_t(1) << 32) - 64) return false;  // 32-bit byte offsets into the planes
    if (s.granularity == SHERRY_PER_TENSOR || s.granularity == SHERRY_PER_CHANNEL) return true;
    if (s.granularity != SHERRY_PER_GROUP) return false;
    return s.group == 128 || s.group == 256;  // K % 512 == 0: 4 or 2 whole groups per unit
}

int64_t stream_tiles(const ProbShape& s) { return (s.N + kSRows - 1) / kSRows; }

// wait budget of the launches (sherry_set_wait_budget)
static std::atomic<long long> g_stream_wait{kSWaitCycles};

long long stream_set_wait_cycles(long long cycles) {
    return g_stream_wait.exchange(cycles > 0 ? cycles : kSWaitCycles);
}

struct SPlan {
    std::vector<SProb> probs;
    int total_units = 0, total_tiles = 0, grid = 0, upc = 0;
    size_t ws_bytes = 0, part_off = 0;
};

static int stream_ctas(int sms) { return sms; }  // one CTA per SM (the stages fill shared memory)

static SPlan make_splan(const ProbShape* shapes, int count, int64_t M, int sms) {
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
    pl.ws_bytes = kTicketBytes + (size_t)pl.grid * 2 * (size_t)M * kSRows * sizeof(float);
    return pl;
}

size_t stream_workspace_bytes(const ProbShape* shapes, int count, int64_t M, int sms) {
    return make_splan(shapes, count, M, sms).ws_bytes;
}

template <int MAXP, int MT>
static int stream_launch_t(SPlan& pl, int y_bf16, void* workspace, cudaStream_t stream) {
    static SParams<MAXP> P;
    static std::mutex mu;
    static PerDevice attr;
    std::lock_guard<std::mutex> lk(mu);
    P.wait_cycles = g_stream_wait.load();
    P.count = (int)pl.probs.size();
    P.y_bf16 = y_bf16;
    P.total_units = pl.total_units;
    P.upc = pl.upc;
    P.ticket = static_cast<int*>(workspace);
    P.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.part_off);
    for (int i = 0; i < P.count; ++i) P.p[i] = pl.probs[i];
    int done = 0;
    const int st = per_device(attr, &done, [](int& v) {
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_lut_stream<MAXP, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               SCfg<MT>::kSmem));
        v = 1;
        return SHERRY_OK;
    });
    if (st) return st;
    k_lut_stream<MAXP, MT><<<pl.grid, kSThreads, SCfg<MT>::kSmem, stream>>>(P);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

template <int MT>
static int stream_launch_mt(SPlan& pl, int count, int y_bf16, void* workspace, cudaStream_t stream) {
    if (count <= 1) return stream_launch_t<1, MT>(pl, y_bf16, workspace, stream);
    if (count <= 16) return stream_launch_t<16, MT>(pl, y_bf16, workspace, stream);
    return stream_launch_t<SHERRY_MAX_BATCH, MT>(pl, y_bf16, workspace, stream);
}

int stream_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                         void* workspace, int sms, cudaStream_t stream) {
    if (M != 1 && M != 2) return SHERRY_ERR_UNSUPPORTED;
    SPlan pl = make_splan(shapes, count, M, sms);
    for (int i = 0; i < count; ++i) {
        SProb& p = pl.probs[i];
        p.X = descs[i].X;
        p.idx = descs[i].idx;
        p.sgn = descs[i].sgn;
        p.scales = descs[i].scales;
        p.Y = descs[i].Y;
    }
    if (pl.total_units == 0) return SHERRY_OK;
    return M == 1 ? stream_launch_mt<1>(pl, count, y_bf16, workspace, stream)
                  : stream_launch_mt<2>(pl, count, y_bf16, workspace, stream);
}

int stream_status_take() {
    int v = 0;
    SHERRY_CUDA_CHECK(cudaMemcpyFromSymbol(&v, g_stream_status, sizeof(int)));
    if (v) {
        const int zero = 0;
        SHERRY_CUDA_CHECK(cudaMemcpyToSymbol(g_stream_status, &zero, sizeof(int)));
    }
    return v;
}

}  // namespace sherry
