// gemv_stream.cu -- packed 3:4 ternary linear for 1 to 16 tokens, streamed from
// HBM: the lookup-table decode for one and two tokens (the method's inference
// scheme: tables built from the activations, looked up by the packed weights,
// accumulated, then scaled; "Sherry: Hardware-Efficient 1.25-Bit Ternary
// Quantization via Fine-grained Sparsification", digest paragraph on inference;
// Y = X T alpha).
//
// Work unit: 512 output rows x 32 W weights (W packed words) of one linear: W =
// 16 for independent linears (one batched launch per decode step) and for
// chained phases of three tokens, W = 8 for a four-token chain (whose tables
// take more shared memory; one- and two-token chains run on whole-K row blocks,
// k_lut_rows, further below).  From three tokens on, independent linears take
// the tensor-core consumers (k_mma_stream, further below) on the same pipeline.
// All units of a phase (one or many independent linears) are split into equal
// contiguous ranges, one per CTA (stream-K): every CTA streams the same number
// of bytes.  A row block whose units straddle CTAs is finished by the CTA that
// arrives last at its ticket, adding the partial sums in CTA order, so Y is
// deterministic.
//
// Phases (chained linears, e.g. the q/k/v -> o -> gate/up -> down projections
// of a decoder layer stack for one token): a later phase may read an earlier
// phase's Y as its X.  The launch is cooperative (one CTA per SM, all resident);
// after its last unit of a phase a CTA adds one arrival to the phase's counter,
// and before building the first tables of a phase a CTA checks (bounded) that
// every CTA has arrived at the previous phase.  Packed weights do not depend on
// X, so the copies of the next units go on while the barrier resolves; a helper
// blocks on it only when the stage it would refill still waits for the blocked
// tables.
//
// Roles (20 warps).  16 consumer warps: each thread owns one row of the unit
// and only looks up and accumulates (per packed word it spreads the 8 nibbles
// and sign bits into two byte-vectors of table offsets, see lut.cuh, and does 8
// lookups per token at the same offsets; alpha is applied once per 128-weight
// group, or once per row).  4 helper warps, one per SM sub-partition: they copy
// each unit's packed planes with cp.async (W/4 lanes read one row's 4W
// contiguous bytes) into an XOR-swizzled ring of stages that the row-per-lane
// reads hit without bank conflicts, and build the unit's 8W tables of 32
// entries per token into the stage's table buffer.  Stages change hands through
// mbarriers; every wait is bounded, and a timeout sets a device status flag
// (reported by sherry_device_status) and ends the CTA.
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
constexpr int kSBars = 128;                        // mbarriers
constexpr int kSHelperThreads = 32 * kSHelpers;
constexpr int kSHelperRows = kSRows / kSHelpers;   // rows each helper warp copies
constexpr int kSRed = 8;                           // split-tile partials loaded at a time
static_assert(kSHelperRows % 32 == 0, "whole rows per helper lane");
// chained launches keep their phase counters at the end of the ticket region
constexpr int kChainCtrs = 512;                    // up to 511 phases + the exit counter
constexpr int kSMaxPhases = kChainCtrs - 1;

// Geometry of a unit of W packed words.
template <int W>
struct SGeo {
    static constexpr int kIdx = kSRows * W * 4;    // packed words of a stage
    static constexpr int kSgn = kSRows * W;        // sign bytes (W per row)
    static constexpr int kSc = kSRows * W;         // scales (at most W/4 floats per row)
    static constexpr int kStage = kIdx + kSgn + kSc;
    static constexpr int kTabs = W * 8;            // tables per unit (one per block of 4 activations)
    static constexpr int kLut = kTabs * kTab;      // one token's tables of a unit
    static constexpr int kRowB = 4 * W;            // packed-word bytes of one row
    static constexpr int kLanesPerRow = W / 4;     // 16-byte chunks per row
    static constexpr int kRowsPerCopy = 32 / kLanesPerRow;
    static constexpr int kSwz = 128 / kRowB;       // rows per 128-byte cycle of the banks
    static_assert(W == 16 || W == 8, "unit widths");
    static_assert(kStage % 256 == 0 && kLut % 256 == 0, "table bases must stay multiples of 256");
    static_assert(kTabs <= kSHelperThreads, "one table per helper thread");
};

// Ring depth and shared bytes for MT tokens and W-word units (tables are
// token-major within a stage): as many stages as fit next to one CTA's
// registers; four tokens take 8-word units (a 16-word stage with their tables
// leaves room for one stage only).
template <int MT, int W>
struct SCfg {
    using G = SGeo<W>;
    static constexpr int kStages =
        W == 16 ? (MT == 1 ? 3 : MT <= 3 ? 2 : 1) : (MT == 1 ? 6 : MT == 2 ? 5 : MT == 3 ? 4 : 3);
    static constexpr int kLutStage = MT * G::kLut;
    static constexpr int kSmem = 256 + kStages * (G::kStage + kLutStage) + kSBars;
    static_assert(kSmem <= 232448, "shared memory per CTA");
    static_assert(kStages >= 2 && kStages <= 6, "ring depth / barrier slots");
};
constexpr long long kSWaitCycles = 4000000000LL;   // default wait budget, ~2 s at the boost clock
// The no-workspace entry point's fixed scratch holds this kernel's largest plan
// (four tokens, one CTA per SM, two partial slots per CTA) on up to 224 SMs.
static_assert(kTicketBytes + (size_t)224 * 2 * 4 * kSRows * sizeof(float) <= SHERRY_NOALLOC_SCRATCH_BYTES,
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
    int count, y_bf16, n_phases;
    float* part;            // [grid][2][MT][kSRows] split-tile partials
    int* ticket;            // [total tiles]
    int* phase_cnt;         // chained launches: [n_phases] arrivals + exit counter; else null
    int ph_unit[MAXP + 1];  // first unit of each phase; ph_unit[n_phases] = all units
    int ph_upc[MAXP];       // units per CTA of each phase
    SProb p[MAXP];
};

// bounded-wait timeouts of this file's kernel (read and cleared by sherry_device_status)
__device__ int g_stream_status = 0;

namespace {

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
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
// non-blocking check that the phase with the given parity completed (the callers spin on it, bounded)
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
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
// As mbar_wait, but each check may suspend the thread in hardware (up to ~10 us)
// until the phase completes instead of returning at once: a waiting warp then
// takes no issue slots from the warps that still work.
__device__ __forceinline__ bool mbar_try_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(10000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                long long budget) {
    if (mbar_try_sleep(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_sleep(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > budget) {
            *abort_flag = 1;
            atomicExch(&g_stream_status, SHERRY_ERR_TIMEOUT);
            return false;
        }
    }
}
// wait until the shared phase counter reaches `target`; false on timeout or abort
__device__ __forceinline__ bool gate_wait(const int* gate, int target, volatile int* abort_flag, long long budget) {
    const volatile int* g = gate;
    if (*g >= target) return true;
    const long long t0 = clock64();
    while (true) {
        if (*g >= target) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > budget) {
            *abort_flag = 1;
            atomicExch(&g_stream_status, SHERRY_ERR_TIMEOUT);
            return false;
        }
    }
}
// arrival at a phase counter: a release at GPU scope (the Y this CTA wrote, seen by
// this thread through the CTA's mbarrier, is visible before the count), no reply
__device__ __forceinline__ void red_release_add(int* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// One warp (all lanes, converged) reads *cnt until it reaches target (every CTA
// arrived at a phase), or once when block is false: 1 = reached, 0 = not yet
// (non-blocking), -1 = timeout or abort.  Lane 0's reads decide for the warp.
__device__ __forceinline__ int grid_poll(const int* cnt, int target, volatile int* abort_flag, long long budget,
                                         bool block, int lane) {
    const long long t0 = clock64();
    while (true) {
        int v = lane == 0 ? ld_acquire(cnt) : 0;
        v = __shfl_sync(kFull, v, 0);
        if (v >= target) return 1;
        if (!block) return 0;
        int quit = 0;
        if (lane == 0) {
            if (*abort_flag) {
                quit = 1;
            } else if (clock64() - t0 > budget) {
                *abort_flag = 1;
                atomicExch(&g_stream_status, SHERRY_ERR_TIMEOUT);
                quit = 1;
            }
        }
        if (__shfl_sync(kFull, quit, 0)) return -1;
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
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

// 8 lookups of one packed word for token TOK: the tables of blocks BOFF..BOFF+7
// sit at shared offsets (BOFF + j) * kTab + TOK * LUT from the addresses in a[],
// whose low byte is the block's table offset -> even-position and odd-position
// partial sums p0 = (v0 + v2) + (v4 + v6), p1 = (v1 + v3) + (v5 + v7), as
// packed pair adds
template <int BOFF, int TOK, int LUT>
__device__ __forceinline__ void token_sums(const uint32_t (&a)[8], float& p0, float& p1) {
    constexpr int T = TOK * LUT;
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
template <int BOFF, int MT, int LUT>
__device__ __forceinline__ void word_sums(uint32_t w, uint32_t s, uint32_t base, float (&p0)[MT], float (&p1)[MT]) {
    uint32_t ev, od;
    spread_word(w, s, ev, od);
    const uint32_t a[8] = {__byte_perm(ev, base, 0x7650u), __byte_perm(od, base, 0x7650u),
                           __byte_perm(ev, base, 0x7651u), __byte_perm(od, base, 0x7651u),
                           __byte_perm(ev, base, 0x7652u), __byte_perm(od, base, 0x7652u),
                           __byte_perm(ev, base, 0x7653u), __byte_perm(od, base, 0x7653u)};
    token_sums<BOFF, 0, LUT>(a, p0[0], p1[0]);
    if constexpr (MT > 1) token_sums<BOFF, 1, LUT>(a, p0[1], p1[1]);
    if constexpr (MT > 2) token_sums<BOFF, 2, LUT>(a, p0[2], p1[2]);
    if constexpr (MT > 3) token_sums<BOFF, 3, LUT>(a, p0[3], p1[3]);
}

struct UnitPos {
    int p, rb, sub;  // problem, row block, sub-slice
};

// the last problem whose first unit is <= u: a binary search, since a CTA's first
// lookup sits on its start-up path and a batch holds up to hundreds of problems
template <int MAXP>
__device__ __forceinline__ UnitPos locate(const SParams<MAXP>& P, int u) {
    int p = 0, hi = P.count - 1;
    while (p < hi) {
        const int mid = (p + hi + 1) >> 1;
        if (P.p[mid].unit_begin <= u)
            p = mid;
        else
            hi = mid - 1;
    }
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

// This CTA's unit range [b, e) of phase ph.
template <int MAXP>
__device__ __forceinline__ void phase_range(const SParams<MAXP>& P, int ph, int& b, int& e) {
    b = P.ph_unit[ph] + (int)blockIdx.x * P.ph_upc[ph];
    e = min(P.ph_unit[ph + 1], b + P.ph_upc[ph]);
}

// The CTA's units in order over all phases (empty phase ranges skipped).
template <int MAXP>
struct UnitCursor {
    int ph, u, e;
    UnitPos pos;
    __device__ __forceinline__ void seek(const SParams<MAXP>& P, int from_ph) {
        for (ph = from_ph; ph < P.n_phases; ++ph) {
            int b;
            phase_range(P, ph, b, e);
            if (b < e) {
                u = b;
                pos = locate(P, u);
                return;
            }
        }
        u = e = 0;
    }
    __device__ __forceinline__ void next(const SParams<MAXP>& P) {
        if (++u < e)
            advance(P.p, pos);
        else
            seek(P, ph + 1);
    }
};

// Copy geometry of helper lane (h, lane) for one row block: the unit's rows
// [Hh, Hh+H), H = kSHelperRows.  Packed words: rows Hh + R*i + lane/C (C = W/4
// lanes per row, R = 32/C rows per copy), 16-byte chunk lane%C of the row's 4W
// bytes, stored at chunk (c ^ ((row / S) % C)) of the row in shared memory, S =
// 128/4W rows per bank cycle (that swizzle term only depends on the lane).  Sign
// bytes and scales: rows Hh + 32i + lane.  Byte offsets from the plane
// bases; a row past N reads row 0 instead (its results are never stored), so
// every copy is in bounds.
template <int W>
struct CopyRows {
    uint32_t idx[kSHelperRows / SGeo<W>::kRowsPerCopy], sgn[kSHelperRows / 32], sc[kSHelperRows / 32];
};

template <int W>
__device__ __forceinline__ void copy_rows(const SProb& pr, int rb, int h, int lane, CopyRows<W>& cr) {
    using G = SGeo<W>;
    const int row0 = rb * kSRows;
#pragma unroll
    for (int i = 0; i < kSHelperRows / G::kRowsPerCopy; ++i) {
        const int row = row0 + kSHelperRows * h + G::kRowsPerCopy * i + lane / G::kLanesPerRow;
        cr.idx[i] = (uint32_t)((int64_t)(row < pr.N ? row : 0) * pr.words * 4 + 16 * (lane % G::kLanesPerRow));
    }
#pragma unroll
    for (int i = 0; i < kSHelperRows / 32; ++i) {
        const int row = row0 + kSHelperRows * h + 32 * i + lane;
        const int rr = row < pr.N ? row : 0;
        cr.sgn[i] = (uint32_t)((int64_t)rr * pr.words);
        cr.sc[i] = (uint32_t)((int64_t)rr * pr.spr * 4);
    }
}

__device__ __forceinline__ const void* byte_off(const void* base, uint32_t off) {
    return static_cast<const char*>(base) + off;
}

// Helper lane's copies of unit (cr's row block, sub-slice `sub`) into `stage`.
template <int W>
__device__ __forceinline__ void copy_unit(const SProb& pr, const CopyRows<W>& cr, int sub, uint32_t stage, int h,
                                          int lane) {
    using G = SGeo<W>;
    constexpr int C = G::kLanesPerRow;
    const char* bi = reinterpret_cast<const char*>(pr.idx) + sub * G::kRowB;
    const uint32_t lrow = (uint32_t)(lane / C);
    const uint32_t di = stage + (uint32_t)(kSHelperRows * h + lrow) * G::kRowB +
                        ((uint32_t)((lane % C) ^ ((lrow / G::kSwz) % C)) << 4);
#pragma unroll
    for (int i = 0; i < kSHelperRows / G::kRowsPerCopy; ++i)
        cp_async16(di + (uint32_t)(G::kRowsPerCopy * G::kRowB * i), byte_off(bi, cr.idx[i]));
    const char* bs = reinterpret_cast<const char*>(pr.sgn) + sub * W;
    const uint32_t ds = stage + G::kIdx + (uint32_t)(kSHelperRows * h + lane) * W;
#pragma unroll
    for (int i = 0; i < kSHelperRows / 32; ++i) {
        if (W == 16)
            cp_async16(ds + 32u * W * i, byte_off(bs, cr.sgn[i]));
        else
            cp_async8(ds + 32u * W * i, byte_off(bs, cr.sgn[i]));
    }
    const uint32_t dc = ds + G::kSgn;
    if (pr.mode == kSG128) {  // W/4 scales per row and unit
        const char* ba = reinterpret_cast<const char*>(pr.scales) + sub * W;
#pragma unroll
        for (int i = 0; i < kSHelperRows / 32; ++i) {
            if (W == 16)
                cp_async16(dc + 32u * W * i, byte_off(ba, cr.sc[i]));
            else
                cp_async8(dc + 32u * W * i, byte_off(ba, cr.sc[i]));
        }
    } else if (pr.mode == kSG256) {  // W/8 scales per row and unit
        const char* ba = reinterpret_cast<const char*>(pr.scales) + sub * (W / 2);
#pragma unroll
        for (int i = 0; i < kSHelperRows / 32; ++i) {
            if (W == 16)
                cp_async8(dc + 32u * W * i, byte_off(ba, cr.sc[i]));
            else
                cp_async4(dc + 32u * W * i, byte_off(ba, cr.sc[i]));
        }
    }
}

// Lookups of one row over the W words of a unit for MT tokens, into u[]; `st`
// and `lut` are shared addresses of the unit's stage and of token 0's tables.
template <int MODE, int MT, int W>
__device__ __forceinline__ void unit_row(uint32_t st, uint32_t lut, int r, float (&u)[MT]) {
    using G = SGeo<W>;
    constexpr int C = G::kLanesPerRow;
    const uint32_t sw = (uint32_t)((r / G::kSwz) % C);
    uint4 sg, av = make_uint4(0u, 0u, 0u, 0u);
    const uint32_t sgn_a = st + G::kIdx + r * W, sc_a = st + G::kIdx + G::kSgn + r * W;
    if (W == 16) {
        sg = lds128(sgn_a);
        if (MODE == kSG128) av = lds128(sc_a);
        if (MODE == kSG256) {
            const uint2 a2 = lds64(sc_a);
            av = make_uint4(a2.x, a2.y, 0u, 0u);
        }
    } else {
        const uint2 s2 = lds64(sgn_a);
        sg = make_uint4(s2.x, s2.y, 0u, 0u);
        if (MODE == kSG128) {
            const uint2 a2 = lds64(sc_a);
            av = make_uint4(a2.x, a2.y, 0u, 0u);
        }
        if (MODE == kSG256) av.x = lds32(sc_a);
    }
    const uint32_t idx_row = st + r * G::kRowB;
#pragma unroll
    for (int m = 0; m < MT; ++m) u[m] = 0.0f;
#pragma unroll
    for (int q = 0; q < C; ++q) {
        const uint4 wq = lds128(idx_row + (((uint32_t)q ^ sw) << 4));
        const uint32_t sq = q == 0 ? sg.x : q == 1 ? sg.y : q == 2 ? sg.z : sg.w;
        const uint32_t tb = lut + (uint32_t)(q * 32 * kTab);  // tables of words 4q..4q+3 (256-aligned)
        float p0[MT], p1[MT], q0[MT], q1[MT], r0[MT], r1[MT], u0[MT], u1[MT];
        word_sums<0, MT, G::kLut>(wq.x, sq & 0xffu, tb, p0, p1);
        word_sums<8, MT, G::kLut>(wq.y, (sq >> 8) & 0xffu, tb, q0, q1);
        word_sums<16, MT, G::kLut>(wq.z, (sq >> 16) & 0xffu, tb, r0, r1);
        word_sums<24, MT, G::kLut>(wq.w, sq >> 24, tb, u0, u1);
        uint32_t ab = 0u;
        if (MODE == kSG128) ab = q == 0 ? av.x : q == 1 ? av.y : q == 2 ? av.z : av.w;
        if (MODE == kSG256) ab = (W == 16 && q >= 2) ? av.y : av.x;
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

template <int MAXP, int MT, int W>
__global__ void __launch_bounds__(kSThreads, 1) k_lut_stream(const __grid_constant__ SParams<MAXP> P) {
    using C = SCfg<MT, W>;
    using G = SGeo<W>;
    constexpr int S = C::kStages;
    __shared__ int s_last;
    __shared__ int s_abort;
    __shared__ int s_gate;  // phases known complete on every CTA (written by helper warp 0)
    // Shared addresses: the buffer is rounded up to 256 bytes, so every table
    // base is a multiple of 256 (a lookup's address replaces its low byte); the
    // XOR swizzles need only 16-byte alignment, since writer and reader apply them.
    const uint32_t stages = (smem_u32(g_smem) + 255u) & ~255u;
    const uint32_t luts = stages + S * G::kStage;  // table buffer s (MT tokens' tables) belongs to stage s
    const uint32_t bars = luts + S * C::kLutStage;
    // ready(s): the stage's planes landed and its tables are built; empty(s): consumers are done with both
    auto ready = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bars + 48u + 8u * (uint32_t)s; };
    const uint32_t bar_part = bars + 96u;    // every consumer stored its split-tile partial
    const uint32_t bar_last = bars + 104u;   // the ticket's outcome is in s_last
    const uint32_t bar_phase = bars + 112u;  // every consumer finished the CTA's units of a phase

    const int t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    const bool chain = P.phase_cnt != nullptr;
    if (t == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(ready(s), kSHelperThreads + G::kTabs);  // a cp.async arrival per helper, one per table
            mbar_init(empty(s), kSRows);
        }
        mbar_init(bar_part, kSRows);
        mbar_init(bar_last, 1);
        mbar_init(bar_phase, kSRows);
        s_abort = 0;
        s_gate = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int* abort_flag = &s_abort;
    // units of this CTA over all phases
    int nu = 0;
    for (int ph = 0; ph < P.n_phases; ++ph) {
        int b, e;
        phase_range(P, ph, b, e);
        nu += max(0, e - b);
    }

    if (warp >= kSConsumers) {
        // ---- helpers: unit j's copies go to stage j % S once the consumers are done
        // with unit j - S there.  Its tables are built right after, unless the unit opens
        // a phase whose input (the previous phase's Y) is not complete yet: then the
        // copies run on and the tables follow once the phase barrier is seen, at the
        // latest before a stage is reused whose consumers need them.
        const int h = warp - kSConsumers;
        const int ht = t - 32 * kSConsumers;  // table (block of 4 activations) of the unit
        const bool tab = ht < G::kTabs;
        UnitCursor<MAXP> cc, tc;              // copy and table cursors
        cc.seek(P, 0);
        tc = cc;
        CopyRows<W> cr;
        int cr_p = -1, cr_rb = -1;
        int passed = 0;       // phases this thread knows complete on every CTA
        int jt = 0;           // units whose tables this thread has built
        bool fail = false;    // a bounded wait gave up
        uint2 xn[MT];         // the activations of the table cursor's unit, loaded one unit ahead
        bool have_x = false;
        // activations: token m's row of X starts K bf16 (words * 8 groups of 4) after
        // token m-1's; read through L2 (a chained phase's X is written by this launch)
        auto load_x = [&](const SProb& px, int sub) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                xn[m] = __ldcg(reinterpret_cast<const uint2*>(px.X) + (int64_t)m * px.words * 8 + sub * G::kTabs + ht);
        };
        // build unit jt's tables; with block == false return false instead of waiting for
        // the phase barrier
        auto tables = [&](bool block) -> bool {
            if (!tab) {  // this thread builds no table: only the cursor moves
                tc.next(P);
                ++jt;
                return true;
            }
            if (chain && tc.ph > passed) {
                // helper warp 0 (as a whole warp) reads the arrivals of every CTA and
                // publishes the phase in a shared counter that the other helper warps read
                // (a monotonic count, so a warp that looks late still sees it)
                if (h == 0) {
                    const int st = grid_poll(P.phase_cnt + tc.ph - 1, (int)gridDim.x, abort_flag, P.wait_cycles,
                                             block, lane);
                    if (st != 1) {
                        fail = st < 0;
                        return false;
                    }
                    __threadfence();
                    if (lane == 0) *reinterpret_cast<volatile int*>(&s_gate) = tc.ph;
                } else if (block) {
                    if (!gate_wait(&s_gate, tc.ph, abort_flag, P.wait_cycles)) {
                        fail = true;
                        return false;
                    }
                } else if (*reinterpret_cast<volatile int*>(&s_gate) < tc.ph) {
                    return false;
                }
                __threadfence();
                passed = tc.ph;
                have_x = false;
            }
            const int s = jt % S;
            if (!have_x) load_x(P.p[tc.pos.p], tc.pos.sub);
#pragma unroll
            for (int m = 0; m < MT; ++m) build_table(luts + s * C::kLutStage + m * G::kLut + ht * kTab, xn[m]);
            mbar_arrive(ready(s));
            tc.next(P);
            ++jt;
            // the next unit's activations are fetched now unless it opens a phase that is
            // still being written
            have_x = jt < nu && (!chain || tc.ph <= passed);
            if (have_x) load_x(P.p[tc.pos.p], tc.pos.sub);
            return true;
        };
        for (int j = 0; j < nu && !fail; ++j) {
            const int s = j % S;
            if (j >= S) {
                // the consumers free stage s after unit j - S, whose tables must exist
                while (jt <= j - S && tables(true)) {
                }
                if (fail || !mbar_wait(empty(s), (uint32_t)(((j / S) & 1) ^ 1), abort_flag, P.wait_cycles)) break;
            }
            const SProb& pr = P.p[cc.pos.p];
            if (cc.pos.p != cr_p || cc.pos.rb != cr_rb) {
                copy_rows<W>(pr, cc.pos.rb, h, lane, cr);
                cr_p = cc.pos.p;
                cr_rb = cc.pos.rb;
            }
            copy_unit<W>(pr, cr, cc.pos.sub, stages + s * G::kStage, h, lane);
            cp_async_arrive(ready(s));
            cc.next(P);
            while (jt <= j && tables(false)) {
            }
        }
        while (!fail && jt < nu && tables(true)) {
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else {
        // ---- consumers: thread t owns row t of every unit
        const int r = t;
        float acc[MT];
        int k = 0;       // units consumed so far (all phases): stage k % S
        int events = 0;  // split tiles handled so far (phase of bar_part / bar_last)
        int phases = 0;  // phases this CTA's consumers completed with units (phase of bar_phase)
        bool ok = true;
        for (int ph = 0; ph < P.n_phases && ok; ++ph) {
            int u_begin, u_end;
            phase_range(P, ph, u_begin, u_end);
            const int pb = P.ph_unit[ph], upc = P.ph_upc[ph];
            if (u_begin < u_end) {
                UnitPos cur = locate(P, u_begin);
                bool tile_from_start = (P.p[cur.p].unit_begin + cur.rb * P.p[cur.p].n_sub == u_begin);
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
                for (int uu = u_begin; uu < u_end; ++uu, ++k) {
                    const int s = k % S;
                    if (!mbar_wait(ready(s), (uint32_t)((k / S) & 1), abort_flag, P.wait_cycles)) {
                        ok = false;
                        break;
                    }
                    const SProb& pr = P.p[cur.p];
                    const uint32_t st = stages + s * G::kStage;
                    const uint32_t lut = luts + s * C::kLutStage;
                    float u[MT];
                    if (pr.mode == kSRow)
                        unit_row<kSRow, MT, W>(st, lut, r, u);
                    else if (pr.mode == kSG128)
                        unit_row<kSG128, MT, W>(st, lut, r, u);
                    else
                        unit_row<kSG256, MT, W>(st, lut, r, u);
#pragma unroll
                    for (int m = 0; m < MT; ++m) acc[m] += u[m];
                    mbar_arrive(empty(s));

                    const bool tile_end = (cur.sub == pr.n_sub - 1);
                    if (tile_end || uu == u_end - 1) {
                        const int n = cur.rb * kSRows + r;
                        const bool row_ok = n < pr.N;
                        float v[MT];
                        const float rs =
                            (pr.mode == kSRow && row_ok) ? __ldg(pr.scales + (pr.per_tensor ? 0 : n)) : 1.0f;
#pragma unroll
                        for (int m = 0; m < MT; ++m) v[m] = pr.mode == kSRow ? acc[m] * rs : acc[m];
                        if (tile_from_start && tile_end) {
                            if (row_ok) {
#pragma unroll
                                for (int m = 0; m < MT; ++m) {
                                    if (P.y_bf16)
                                        reinterpret_cast<__nv_bfloat16*>(pr.Y)[(int64_t)m * pr.N + n] =
                                            __float2bfloat16_rn(v[m]);
                                    else
                                        reinterpret_cast<float*>(pr.Y)[(int64_t)m * pr.N + n] = v[m];
                                }
                            }
                        } else {
                            // split tile: partials into this CTA's slot, then the ticket
                            const int tile = pr.tile_begin + cur.rb;
                            const int tile_u0 = pr.unit_begin + cur.rb * pr.n_sub;
                            const int c_a = (tile_u0 - pb) / upc;
                            const int c_b = (tile_u0 + pr.n_sub - 1 - pb) / upc;
                            const int slot = (u_begin >= tile_u0) ? 0 : 1;
#pragma unroll
                            for (int m = 0; m < MT; ++m)
                                __stcg(P.part + (((int64_t)blockIdx.x * 2 + slot) * MT + m) * kSRows + r, v[m]);
                            __threadfence();
                            mbar_arrive(bar_part);
                            const uint32_t ph2 = (uint32_t)(events & 1);
                            ++events;
                            // every consumer waits for all partials (no lane of a warp spins on
                            // another barrier than its neighbours: divergent spins can starve)
                            const bool stored = mbar_wait(bar_part, ph2, abort_flag, P.wait_cycles);
                            if (stored && r == 0) {
                                s_last = (atomicAdd(P.ticket + tile, 1) == c_b - c_a);
                                mbar_arrive(bar_last);
                            }
                            __syncwarp();
                            if (!stored || !mbar_wait(bar_last, ph2, abort_flag, P.wait_cycles)) {
                                ok = false;
                                break;
                            }
                            if (s_last) {
                                __threadfence();
                                // the partials of CTAs c_a..c_b added in CTA order; their loads are
                                // issued kSRed at a time (a chained phase splits a tile over up to
                                // 32 CTAs, and one dependent L2 round trip each would dominate it)
                                float sums[MT];
#pragma unroll
                                for (int m = 0; m < MT; ++m) sums[m] = 0.0f;
                                for (int c0 = c_a; c0 <= c_b; c0 += kSRed) {
                                    float pv[kSRed][MT];
#pragma unroll
                                    for (int i = 0; i < kSRed; ++i) {
                                        const int c = c0 + i;
                                        const int sl = (pb + c * upc >= tile_u0) ? 0 : 1;
#pragma unroll
                                        for (int m = 0; m < MT; ++m)
                                            pv[i][m] = c <= c_b ? __ldcg(P.part + (((int64_t)c * 2 + sl) * MT + m) * kSRows + r)
                                                                : 0.0f;
                                    }
#pragma unroll
                                    for (int i = 0; i < kSRed; ++i)
#pragma unroll
                                        for (int m = 0; m < MT; ++m)
                                            if (c0 + i <= c_b) sums[m] = (c0 + i == c_a) ? pv[i][m] : sums[m] + pv[i][m];
                                }
#pragma unroll
                                for (int m = 0; m < MT; ++m) {
                                    const float sum = sums[m];
                                    if (row_ok) {
                                        if (P.y_bf16)
                                            reinterpret_cast<__nv_bfloat16*>(pr.Y)[(int64_t)m * pr.N + n] =
                                                __float2bfloat16_rn(sum);
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
                if (!ok) break;
                if (chain) {
                    // every consumer's Y of this phase is written before the CTA's arrival;
                    // warp 0 waits for all of them (as a whole warp) and lane 0 arrives
                    __threadfence();
                    mbar_arrive(bar_phase);
                    if (warp == 0) {
                        const bool done = mbar_wait(bar_phase, (uint32_t)(phases & 1), abort_flag, P.wait_cycles);
                        if (done && lane == 0) red_release_add(P.phase_cnt + ph, 1);
                        __syncwarp();
                        if (!done) {
                            ok = false;
                            break;
                        }
                    }
                    ++phases;
                }
            } else if (chain && r == 0) {
                red_release_add(P.phase_cnt + ph, 1);  // nothing of this phase here
            }
        }
    }

    __syncthreads();
    if (chain && t == 0 && !*abort_flag) {
        // the last CTA to leave zeroes the phase counters for the next launch
        __threadfence();
        if (atomicAdd(P.phase_cnt + P.n_phases, 1) == (int)gridDim.x - 1) {
            for (int ph = 0; ph <= P.n_phases; ++ph) P.phase_cnt[ph] = 0;
            __threadfence();
        }
    }
}

// ---- tensor-core consumers for 4 to 16 tokens ------------------------------------
//
// The same streaming pipeline (units of 512 rows x 512 weights, stream-K ranges,
// helper warps copying the packed planes into a cp.async ring, split tiles
// finished through tickets), with a different consumer: instead of one table
// lookup per block and token, each 4-weight block is expanded once to bf16
// {-1, 0, +1} (two 4-byte lookups in a 32-entry pattern table) straight into the
// A fragment of mma.sync m16n8k16 and multiplied with all tokens at once.  The
// helpers stage the unit's activations (NT token rows of 512 bf16, zero rows for
// tokens >= M) in the stage instead of tables.  K is permuted inside each 32-weight
// word identically for both operands: in slice h of a word the lane with c =
// lane % 4 holds the fragment positions k = 2c, 2c+1, 2c+8, 2c+9, taken to be the 4
// weights of block 2c + h, so its two blocks per word are byte c of the packed
// word and its activation fragments for both slices are the 8 consecutive
// activations 8c .. 8c+7 of the word, one 16-byte load.  A lane gathers byte c of
// the four words of a row's 16-byte chunk into one register and spreads all eight
// blocks into table offsets at once; each block then costs one byte permute (its
// table address) and the two lookups.  Each consumer warp owns
// 32 rows (two m16 tiles); alpha is applied once per scale group (or at the end
// for row scales) in fp32 registers.

constexpr int kMXRow = 16 * 32 * 2 + 64;  // bytes per staged token row (padded: conflict-free 16-byte reads)
constexpr int kMPat = 256;                // pattern table: 32 low words (weights 0, 1), then 32 high words

// The no-workspace entry point's fixed scratch holds the largest tensor-core plan
// (sixteen tokens, one CTA per SM, two partial slots per CTA) on up to 224 SMs.
static_assert(kTicketBytes + (size_t)224 * 2 * 16 * kSRows * sizeof(float) <= SHERRY_NOALLOC_SCRATCH_BYTES,
              "no-workspace scratch too small for the tensor-core streaming plan");

template <int NT>
struct MCfg {
    using G = SGeo<16>;
    static constexpr int kStages = 3;
    static constexpr int kX = NT * kMXRow;  // staged activations per stage
    static constexpr int kStage = G::kStage + kX;
    static constexpr int kSmem = 256 + kMPat + kStages * kStage + kSBars;
    static_assert(kSmem <= 232448, "shared memory per CTA");
    static_assert(kStage % 16 == 0, "16-byte aligned stages");
};

__device__ __forceinline__ void m_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Table offsets of the lane's blocks in the four words of a 16-byte chunk: byte j of
// ev is 4 * code of block 2c of word j, of od of block 2c + 1 (code = nibble + 16 G;
// s holds the four words' sign bytes).  Byte c of every word is gathered first
// (gsel = c | (c + 4) << 4), so one spread serves the four words; the sign bits 2c
// and 2c + 1 of each sign byte move to bit 6 with one shift (gsh = 6 - 2c).
__device__ __forceinline__ void m_offsets(uint4 w, uint32_t s, uint32_t gsel, uint32_t gsh, uint32_t& ev,
                                          uint32_t& od) {
    const uint32_t b = __byte_perm(__byte_perm(w.x, w.y, gsel), __byte_perm(w.z, w.w, gsel), 0x5410u);
    const uint32_t v = s << gsh;
    ev = ((b << 2) & 0x3c3c3c3cu) | (v & 0x40404040u);
    od = ((b >> 2) & 0x3c3c3c3cu) | ((v >> 1) & 0x40404040u);
}

template <int MAXP, int NT>
__global__ void __launch_bounds__(kSThreads, 1) k_mma_stream(const __grid_constant__ SParams<MAXP> P, int M) {
    using C = MCfg<NT>;
    using G = SGeo<16>;
    constexpr int S = C::kStages;
    constexpr int NB = NT / 8;  // n8 token tiles
    __shared__ int s_last;
    __shared__ int s_abort;
    const uint32_t base = (smem_u32(g_smem) + 255u) & ~255u;
    const uint32_t pat = base;                     // [32] low words, [32] high words
    const uint32_t stages = base + kMPat;          // stage s: planes, then NT staged token rows
    const uint32_t bars = stages + S * C::kStage;
    auto ready = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bars + 48u + 8u * (uint32_t)s; };
    const uint32_t bar_part = bars + 96u;
    const uint32_t bar_last = bars + 104u;

    const int t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    if (t == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(ready(s), kSHelperThreads + kSHelperThreads);  // a cp.async and a staging arrival per helper
            mbar_init(empty(s), kSRows);
        }
        mbar_init(bar_part, kSRows);
        mbar_init(bar_last, 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (t < 32) {
        const uint2 e = decode_block_bf16(t & 15u, t >> 4);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(pat + 4u * t), "r"(e.x) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(pat + 128u + 4u * t), "r"(e.y) : "memory");
    }
    // token rows >= M read zeros: written once, never copied over
    for (int i = t; i < S * (NT - M) * (kMXRow / 16); i += kSThreads) {
        const int per = (NT - M) * (kMXRow / 16);
        const int s = i / per, r = i % per;
        const int m = M + r / (kMXRow / 16), ch = r % (kMXRow / 16);
        sts128(stages + s * C::kStage + G::kStage + m * kMXRow + 16 * ch, make_uint4(0u, 0u, 0u, 0u));
    }
    __syncthreads();
    volatile int* abort_flag = &s_abort;
    int u_begin, u_end;
    phase_range(P, 0, u_begin, u_end);
    const int nu = max(0, u_end - u_begin);

    if (warp >= kSConsumers) {
        // ---- helpers: copies and activation staging of unit j into stage j % S
        const int h = warp - kSConsumers;
        const int ht = t - 32 * kSConsumers;
        UnitPos cu = locate(P, u_begin);
        CopyRows<16> cr;
        int cr_p = -1, cr_rb = -1;
        for (int j = 0; j < nu; ++j) {
            const int s = j % S;
            if (j >= S && !mbar_wait(empty(s), (uint32_t)(((j / S) & 1) ^ 1), abort_flag, P.wait_cycles)) break;
            const SProb& pr = P.p[cu.p];
            if (cu.p != cr_p || cu.rb != cr_rb) {
                copy_rows<16>(pr, cu.rb, h, lane, cr);
                cr_p = cu.p;
                cr_rb = cu.rb;
            }
            const uint32_t st = stages + s * C::kStage;
            copy_unit<16>(pr, cr, cu.sub, st, h, lane);
            cp_async_arrive(ready(s));
            // the unit's 512 activations of each token (64 chunks of 16 bytes per token)
            const uint4* xs = reinterpret_cast<const uint4*>(pr.X) + (int64_t)cu.sub * 64;
            for (int i = ht; i < M * 64; i += kSHelperThreads) {
                const int m = i >> 6, ch = i & 63;
                sts128(st + G::kStage + m * kMXRow + 16 * ch, __ldg(xs + (int64_t)m * pr.words * 4 + ch));
            }
            mbar_arrive(ready(s));
            advance(P.p, cu);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        return;
    }

    // ---- consumers: warp w owns unit rows 32w .. 32w+31 as two m16 tiles
    const int g = lane >> 2, c = lane & 3;
    const uint32_t gsel = (uint32_t)c | ((uint32_t)(c + 4) << 4), gsh = 6u - 2u * (uint32_t)c;
    int rows[4];  // unit rows of the lane: tile 0 rows g, g+8; tile 1 rows g, g+8
#pragma unroll
    for (int i = 0; i < 4; ++i) rows[i] = 32 * warp + 16 * (i >> 1) + g + 8 * (i & 1);
    float acc[2][NB][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[a][b][i] = 0.0f;
    UnitPos cur = locate(P, u_begin);
    bool tile_from_start = (P.p[cur.p].unit_begin + cur.rb * P.p[cur.p].n_sub == u_begin);
    const int pb = P.ph_unit[0], upc = P.ph_upc[0];
    int events = 0;
    for (int k = 0; k < nu; ++k) {
        const int s = k % S;
        if (!mbar_wait(ready(s), (uint32_t)((k / S) & 1), abort_flag, P.wait_cycles)) break;
        const SProb& pr = P.p[cur.p];
        const uint32_t st = stages + s * C::kStage;
        const uint32_t xs = st + G::kStage + (uint32_t)(g * kMXRow + 16 * c);
        const int mode = pr.mode;
        float cs[2][NB][4];  // group partial sums: row tile, token tile
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (q == 0 || mode == kSG128 || (mode == kSG256 && q == 2)) {
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int b = 0; b < NB; ++b)
#pragma unroll
                        for (int i = 0; i < 4; ++i) cs[a][b][i] = 0.0f;
            }
            // rows' packed words: each lane reads its rows' 4-word chunk and spreads its
            // blocks of all four words into table offsets at once (m_offsets)
            uint32_t evr[4], odr[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = rows[i];
                const uint32_t chunk = st + r * G::kRowB + (((uint32_t)q ^ (uint32_t)((r / G::kSwz) % G::kLanesPerRow)) << 4);
                m_offsets(lds128(chunk), lds32(st + G::kIdx + r * 16 + 4 * q), gsel, gsh, evr[i], odr[i]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 xb[NB];
#pragma unroll
                for (int b = 0; b < NB; ++b) xb[b] = lds128(xs + (uint32_t)(b * 8 * kMXRow + (4 * q + j) * 64));
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    uint32_t A[2][2][2];  // row of the tile, slice, (low, high)
#pragma unroll
                    for (int ii = 0; ii < 2; ++ii) {
                        const int i = 2 * a + ii;
                        // table addresses of blocks 2c and 2c + 1 of word j (the table base
                        // is 256-byte aligned: its low byte is the offset)
                        const uint32_t aa = __byte_perm(evr[i], pat, 0x7650u | (uint32_t)j);
                        const uint32_t ab = __byte_perm(odr[i], pat, 0x7650u | (uint32_t)j);
                        A[ii][0][0] = lds32(aa);
                        A[ii][0][1] = lds32(aa + 128u);
                        A[ii][1][0] = lds32(ab);
                        A[ii][1][1] = lds32(ab + 128u);
                    }
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int b = 0; b < NB; ++b) {
                            const uint32_t b0 = hh ? xb[b].z : xb[b].x, b1 = hh ? xb[b].w : xb[b].y;
                            m_mma(cs[a][b], A[0][hh][0], A[1][hh][0], A[0][hh][1], A[1][hh][1], b0, b1);
                        }
                }
            }
            // end of a scale group (group 128: every 4 words; 256: every 8; row scales: the unit)
            if (mode == kSG128 || (mode == kSG256 && (q & 1)) || (mode == kSRow && q == 3)) {
                float al[4] = {1.0f, 1.0f, 1.0f, 1.0f};
                if (mode != kSRow) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t sc_a = st + G::kIdx + G::kSgn + rows[i] * 16;
                        al[i] = __uint_as_float(lds32(mode == kSG128 ? sc_a + 4 * q : sc_a + 4 * (q >> 1)));
                    }
                }
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int b = 0; b < NB; ++b)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float v = cs[a][b][i];
                            acc[a][b][i] = mode == kSRow ? acc[a][b][i] + v : fmaf(al[2 * a + (i >> 1)], v, acc[a][b][i]);
                        }
            }
        }
        mbar_arrive(empty(s));

        const bool tile_end = (cur.sub == pr.n_sub - 1);
        if (tile_end || k == nu - 1) {
            // lane values: acc[a][b][i] = row rows[2a + (i >> 1)], token 8b + 2c + (i & 1)
            float v[2][NB][4];
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int n = cur.rb * kSRows + rows[2 * a + (i >> 1)];
                    const float rs = (pr.mode == kSRow && n < pr.N) ? __ldg(pr.scales + (pr.per_tensor ? 0 : n)) : 1.0f;
#pragma unroll
                    for (int b = 0; b < NB; ++b) v[a][b][i] = pr.mode == kSRow ? acc[a][b][i] * rs : acc[a][b][i];
                }
            auto store = [&](int a, int b, int i, float val) {
                const int n = cur.rb * kSRows + rows[2 * a + (i >> 1)];
                const int m = 8 * b + 2 * c + (i & 1);
                if (n < pr.N && m < M) {
                    if (P.y_bf16)
                        reinterpret_cast<__nv_bfloat16*>(pr.Y)[(int64_t)m * pr.N + n] = __float2bfloat16_rn(val);
                    else
                        reinterpret_cast<float*>(pr.Y)[(int64_t)m * pr.N + n] = val;
                }
            };
            if (tile_from_start && tile_end) {
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int b = 0; b < NB; ++b)
#pragma unroll
                        for (int i = 0; i < 4; ++i) store(a, b, i, v[a][b][i]);
            } else {
                // split tile: partials [cta][slot][token][row], then the ticket
                const int tile = pr.tile_begin + cur.rb;
                const int tile_u0 = pr.unit_begin + cur.rb * pr.n_sub;
                const int c_a = (tile_u0 - pb) / upc;
                const int c_b = (tile_u0 + pr.n_sub - 1 - pb) / upc;
                const int slot = (u_begin >= tile_u0) ? 0 : 1;
                auto part = [&](int cta, int sl, int a, int b, int i) {
                    const int m = 8 * b + 2 * c + (i & 1);
                    return P.part + (((int64_t)cta * 2 + sl) * M + m) * kSRows + rows[2 * a + (i >> 1)];
                };
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int b = 0; b < NB; ++b)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            if (8 * b + 2 * c + (i & 1) < M) __stcg(part((int)blockIdx.x, slot, a, b, i), v[a][b][i]);
                __threadfence();
                mbar_arrive(bar_part);
                const uint32_t ph2 = (uint32_t)(events & 1);
                ++events;
                const bool stored = mbar_wait(bar_part, ph2, abort_flag, P.wait_cycles);
                if (stored && t == 0) {
                    s_last = (atomicAdd(P.ticket + tile, 1) == c_b - c_a);
                    mbar_arrive(bar_last);
                }
                __syncwarp();
                if (!stored || !mbar_wait(bar_last, ph2, abort_flag, P.wait_cycles)) break;
                if (s_last) {
                    __threadfence();
#pragma unroll
                    for (int a = 0; a < 2; ++a)
#pragma unroll
                        for (int b = 0; b < NB; ++b)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                if (8 * b + 2 * c + (i & 1) >= M) continue;
                                float sum = 0.0f;
                                for (int cc = c_a; cc <= c_b; ++cc) {
                                    const int sl = (pb + cc * upc >= tile_u0) ? 0 : 1;
                                    const float pv = __ldcg(part(cc, sl, a, b, i));
                                    sum = (cc == c_a) ? pv : sum + pv;
                                }
                                store(a, b, i, sum);
                            }
                    if (t == 0) P.ticket[tile] = 0;  // leave the ticket zeroed
                }
            }
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[a][b][i] = 0.0f;
            tile_from_start = true;
        }
        advance(P.p, cur);
    }
}

// ---- chained decode on whole-K row blocks (one and two tokens) ---------------------
//
// A chained phase of one decode step holds 4.5-19 MB of packed weights; split into
// the streaming kernel's 512 x 512 units, every row block of a phase is shared by
// 6-16 CTAs and each phase pays the split-tile handshake (partials, ticket, the last
// CTA's sum) on top of the grid barrier.  This kernel gives every row block to one
// CTA instead.  Item = 32 rows of one linear over all of K: lane = row, and the 16
// consumer warps split K into 128-weight slices (one packed 16-byte chunk, one
// group-128 scale), so the K reduction stays inside the CTA (a fixed-order sum
// over the warps in shared memory).  K runs in chunks of 24 slices (3072 weights)
// for one token and 16 slices for two (their tables take twice the space): per
// chunk the consumers build the chunk's tables (one or two per thread and token;
// a warp takes slices w and w + 16) and then look up every item of the CTA's
// current segment (up to kCSeg items of one linear), so the tables are built once
// per segment, not per item, and a K of 3072 is one chunk.  Four
// helper warps copy the items' packed words (row-major, XOR-swizzled 16-byte
// chunks), sign words and scales (rows padded by 16 bytes) with 16-byte copies
// into a ring of stages; they run ahead across phases, since weights do not
// depend on X.  Each phase's items are split into contiguous, balanced ranges over
// the CTAs; a CTA arrives at the phase counter after its Y stores (release) and
// waits for the previous phase's count before reading its X (acquire).  The next
// chunk's X is loaded during the current chunk's lookups, and waiting warps suspend
// on their mbarrier instead of polling, so they leave the issue slots to the
// working ones.
constexpr int kCRows = 32;                      // rows per item: one per lane
constexpr int kCSeg = 4;                        // items of one linear sharing the tables
constexpr int kCStages = 4;

// Chunk geometry and shared memory for MT tokens.
template <int MT>
struct CCfg {
    static constexpr int kSl = MT == 1 ? 24 : 16;        // 128-weight slices per chunk (warp w: w, w + 16)
    static constexpr int kChunk = 128 * kSl;              // weights per chunk
    static constexpr int kBlocks = kChunk / 4;            // tables per chunk and token
    static constexpr int kTPT = (kBlocks + kSRows - 1) / kSRows;  // tables per consumer thread
    static constexpr int kIdx = kCRows * kSl * 16;        // packed words of a stage: [row][slice] 16-byte chunks
    static constexpr int kPad = 4 * kSl + 16;             // bytes per row of sign words or scales (padded)
    static constexpr int kSgn = kCRows * kPad;            // sign words: 4 sign bytes per slice
    static constexpr int kSc = kCRows * kPad;             // scales: one per slice (group 128) or per two (256)
    static constexpr int kStage = kIdx + kSgn + kSc;
    static constexpr int kTok = kBlocks * kTab;           // one token's tables of a chunk
    static constexpr int kStages = MT * kTok;             // after the tables
    static constexpr int kRed = kStages + kCStages * kStage;  // [warp][item][token][row] partials
    static constexpr int kBars = kRed + kSConsumers * kCSeg * MT * kCRows * 4;
    static constexpr int kSmem = 256 + kBars + 8 * (2 * kCStages + 1);
    static_assert(kSmem <= 232448, "shared memory per CTA");
    static_assert(kSl % 8 == 0 && kSl <= 2 * kSConsumers, "whole swizzle groups; at most two slices per warp");
    static_assert(kTok % 256 == 0 && (32 * kTab) % 256 == 0, "256-aligned table bases");
    static_assert(kStage % 16 == 0 && kIdx % 16 == 0 && kPad % 16 == 0, "16-byte aligned copies");
};

struct CProb {
    const uint16_t* X;
    const uint32_t* idx;
    const uint8_t* sgn;
    const float* scales;
    void* Y;
    int N, K, spr;      // spr: scales per row (group scales)
    int mode, per_tensor;
    int n_items, item_begin;  // 32-row items; the first one's index in the launch
};

template <int MAXP>
struct CParams {
    long long wait_cycles;
    int count, y_bf16, n_phases;
    int* phase_cnt;          // [n_phases] arrivals + the exit counter
    int ph_prob[MAXP + 1];   // first problem of each phase
    int ph_item[MAXP + 1];   // first item of each phase; ph_item[n_phases] = all items
    CProb p[MAXP];
};

struct CSeg {
    int p, it, n;  // problem, its first item of the segment, items
};

// the segment of this CTA's range [g, e) of a phase that starts at launch item g
template <int MAXP>
__device__ __forceinline__ CSeg seg_at(const CParams<MAXP>& P, int ph, int g, int e) {
    int lo = P.ph_prob[ph], hi = P.ph_prob[ph + 1] - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.p[mid].item_begin <= g)
            lo = mid;
        else
            hi = mid - 1;
    }
    const CProb& pr = P.p[lo];
    return CSeg{lo, g - pr.item_begin, min(kCSeg, min(e, pr.item_begin + pr.n_items) - g)};
}

template <int MAXP>
__device__ __forceinline__ void cta_items(const CParams<MAXP>& P, int ph, int& b, int& e) {
    const int b0 = P.ph_item[ph];
    const long long n = P.ph_item[ph + 1] - b0;
    b = b0 + (int)(n * blockIdx.x / gridDim.x);
    e = b0 + (int)(n * (blockIdx.x + 1) / gridDim.x);
}

template <int MT>
__device__ __forceinline__ int chunk_slices(const CProb& pr, int c) {
    return min(CCfg<MT>::kSl, (pr.K - c * CCfg<MT>::kChunk) >> 7);
}

// Copy item `it`, chunk c of problem pr into the stage at st (128 helper threads,
// ht = 0..127); rows past N are not copied (their results are never stored).
template <int MT>
__device__ __forceinline__ void copy_item(const CProb& pr, int it, int c, uint32_t st, int ht) {
    using C = CCfg<MT>;
    const int row0 = it * kCRows;
    const int rows = min(kCRows, pr.N - row0);
    const int nsl = chunk_slices<MT>(pr, c);
    const char* ib = reinterpret_cast<const char*>(pr.idx) + (int64_t)row0 * (pr.K >> 3) + (c * C::kChunk >> 3);
    for (int i = ht; i < rows * nsl; i += kSHelperThreads) {
        const int r = i / nsl, q = i - r * nsl;
        cp_async16(st + r * (16 * C::kSl) + ((q ^ (r & 7)) << 4), ib + (int64_t)r * (pr.K >> 3) + 16 * q);
    }
    // sign words: 4 * nsl bytes per row, whole 16-byte pieces (nsl is a multiple of 4)
    const char* sb = reinterpret_cast<const char*>(pr.sgn) + (int64_t)row0 * (pr.K >> 5) + (c * C::kChunk >> 5);
    const int sp = nsl >> 2;
    for (int i = ht; i < rows * sp; i += kSHelperThreads) {
        const int r = i / sp, q = i - r * sp;
        cp_async16(st + C::kIdx + r * C::kPad + 16 * q, sb + (int64_t)r * (pr.K >> 5) + 16 * q);
    }
    if (pr.mode != kSRow) {
        // group 128: nsl scales per row (16-byte pieces); group 256: nsl / 2 (8-byte pieces)
        const int bytes = pr.mode == kSG128 ? 4 * nsl : 2 * nsl;
        const char* cb = reinterpret_cast<const char*>(pr.scales + (int64_t)row0 * pr.spr) +
                         (pr.mode == kSG128 ? 4 * c * C::kSl : 2 * c * C::kSl);
        const uint32_t sc = st + C::kIdx + C::kSgn;
        if (pr.mode == kSG128) {
            const int np = bytes >> 4;
            for (int i = ht; i < rows * np; i += kSHelperThreads) {
                const int r = i / np, q = i - r * np;
                cp_async16(sc + r * C::kPad + 16 * q, cb + (int64_t)r * 4 * pr.spr + 16 * q);
            }
        } else {
            const int np = bytes >> 3;
            for (int i = ht; i < rows * np; i += kSHelperThreads) {
                const int r = i / np, q = i - r * np;
                cp_async8(sc + r * C::kPad + 8 * q, cb + (int64_t)r * 4 * pr.spr + 8 * q);
            }
        }
    }
}

__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

template <int MAXP, int MT>
__global__ void __launch_bounds__(kSThreads, 1) k_lut_rows(const __grid_constant__ CParams<MAXP> P) {
    using C = CCfg<MT>;
    constexpr int S = kCStages;
    __shared__ int s_abort;
    const uint32_t tabs = (smem_u32(g_smem) + 255u) & ~255u;  // [token][C::kBlocks tables]
    const uint32_t stages = tabs + C::kStages;
    const uint32_t red = tabs + C::kRed;
    const uint32_t bars = tabs + C::kBars;
    auto ready = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bars + 8u * (uint32_t)(S + s); };
    const uint32_t cb = bars + 8u * (uint32_t)(2 * S);  // the consumer warps' own barrier

    const int t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    if (t == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(ready(s), kSHelperThreads);  // one cp.async arrival per helper thread
            mbar_init(empty(s), kSConsumers);      // one arrival per consumer warp
        }
        mbar_init(cb, kSConsumers);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int* abort_flag = &s_abort;

    if (warp >= kSConsumers) {
        // ---- helpers: the CTA's stages (segment, chunk, item) in the consumers' order
        const int ht = t - 32 * kSConsumers;
        int j = 0;
        bool ok = true;
        for (int ph = 0; ph < P.n_phases && ok; ++ph) {
            int b, e;
            cta_items(P, ph, b, e);
            for (int g = b; g < e && ok;) {
                const CSeg sg = seg_at(P, ph, g, e);
                const CProb& pr = P.p[sg.p];
                const int nc = (pr.K + C::kChunk - 1) / C::kChunk;
                for (int c = 0; c < nc && ok; ++c)
                    for (int i = 0; i < sg.n; ++i, ++j) {
                        const int s = j % S;
                        if (j >= S && !mbar_wait_sleep(empty(s), (uint32_t)(((j / S) & 1) ^ 1), abort_flag, P.wait_cycles)) {
                            ok = false;
                            break;
                        }
                        copy_item<MT>(pr, sg.it + i, c, stages + s * C::kStage, ht);
                        cp_async_arrive(ready(s));
                    }
                g += sg.n;
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else {
        // ---- consumers: lane = row of the item, warp w = 128-weight slices w and w + 16
        // of the chunk
        const int w = warp, r = lane;
        int k = 0;   // stages consumed
        int nb = 0;  // consumer barriers passed
        bool ok = true;
        // a barrier of the 16 consumer warps: each warp's lanes meet first, then lane 0
        // arrives for the warp (its release covers the lanes' shared-memory writes)
        auto csync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(cb);
            const bool fine = mbar_wait_sleep(cb, (uint32_t)(nb & 1), abort_flag, P.wait_cycles);
            ++nb;
            return fine;
        };
        float acc[kCSeg][MT];
        uint2 xn[C::kTPT][MT];  // this thread's blocks of the next chunk's activations, per token
        // activations of blocks t and t + 512 of chunk c (read through L2: an earlier
        // phase of this launch wrote them)
        auto load_x = [&](const CProb& px, int c) {
            const uint2* xs = reinterpret_cast<const uint2*>(px.X) + (c * C::kChunk >> 2) + t;
            const int nb4 = 32 * chunk_slices<MT>(px, c);
#pragma unroll
            for (int u = 0; u < C::kTPT; ++u)
                if (t + kSRows * u < nb4) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) xn[u][m] = __ldcg(xs + kSRows * u + (int64_t)m * (px.K >> 2));
                }
        };
        for (int ph = 0; ph < P.n_phases && ok; ++ph) {
            int b, e;
            cta_items(P, ph, b, e);
            bool gated = ph == 0;
            bool have_x = false;  // xn holds the next chunk's activations
            for (int g = b; g < e && ok;) {
                const CSeg sg = seg_at(P, ph, g, e);
                const CProb& pr = P.p[sg.p];
                const int nc = (pr.K + C::kChunk - 1) / C::kChunk;
#pragma unroll
                for (int i = 0; i < kCSeg; ++i)
#pragma unroll
                    for (int m = 0; m < MT; ++m) acc[i][m] = 0.0f;
                for (int c = 0; c < nc && ok; ++c) {
                    if (!gated) {
                        // every CTA is past the previous phase: this phase's X is complete.  Lane 0's
                        // acquire read orders the producers' Y stores before its own later
                        // operations, and its arrival at the consumer barrier below (a release at
                        // CTA scope) before every warp's X reads, so no fence is needed here.
                        if (w == 0) {
                            if (grid_poll(P.phase_cnt + ph - 1, (int)gridDim.x, abort_flag, P.wait_cycles, true,
                                          lane) != 1) {
                                ok = false;
                                break;
                            }
                        }
                        gated = true;
                    }
                    // nobody reads the tables any more and, after a grid barrier, every warp
                    // may read the new X
                    if (!(ok = csync())) break;
                    const uint32_t tb0 = tabs;
                    const int nsl = chunk_slices<MT>(pr, c);
                    if (!have_x) load_x(pr, c);
#pragma unroll
                    for (int u = 0; u < C::kTPT; ++u)
                        if (t + kSRows * u < 32 * nsl) {
#pragma unroll
                            for (int m = 0; m < MT; ++m)
                                build_table(tb0 + m * C::kTok + (t + kSRows * u) * kTab, xn[u][m]);
                        }
                    // the next chunk's activations load while this one is looked up: the next
                    // chunk of this linear, or the first of the CTA's next segment in this phase
                    // (its X is complete too)
                    have_x = true;
                    if (c + 1 < nc)
                        load_x(pr, c + 1);
                    else if (g + sg.n < e)
                        load_x(P.p[seg_at(P, ph, g + sg.n, e).p], 0);
                    else
                        have_x = false;
                    if (!(ok = csync())) break;
#pragma unroll
                    for (int i = 0; i < kCSeg; ++i) {
                        if (i < sg.n) {
                            const int s = k % S;
                            if (!(ok = mbar_wait_sleep(ready(s), (uint32_t)((k / S) & 1), abort_flag, P.wait_cycles))) break;
                            const uint32_t st = stages + s * C::kStage;
#pragma unroll
                            for (int h = 0; h < C::kSl; h += kSConsumers) {
                                const int sl = w + h;  // this warp's slice
                                if (sl < nsl) {
                                    const uint4 wq = lds128(st + r * (16 * C::kSl) +
                                                            (((uint32_t)sl ^ (uint32_t)(r & 7)) << 4));
                                    const uint32_t sq = lds32(st + C::kIdx + r * C::kPad + 4 * sl);
                                    const uint32_t tb = tb0 + (uint32_t)(sl * 32 * kTab);
                                    float p0[MT], p1[MT], q0[MT], q1[MT], r0[MT], r1[MT], u0[MT], u1[MT];
                                    word_sums<0, MT, C::kTok>(wq.x, sq & 0xffu, tb, p0, p1);
                                    word_sums<8, MT, C::kTok>(wq.y, (sq >> 8) & 0xffu, tb, q0, q1);
                                    word_sums<16, MT, C::kTok>(wq.z, (sq >> 16) & 0xffu, tb, r0, r1);
                                    word_sums<24, MT, C::kTok>(wq.w, sq >> 24, tb, u0, u1);
                                    float al = 1.0f;
                                    if (pr.mode == kSG128)
                                        al = __uint_as_float(lds32(st + C::kIdx + C::kSgn + r * C::kPad + 4 * sl));
                                    if (pr.mode == kSG256)
                                        al = __uint_as_float(lds32(st + C::kIdx + C::kSgn + r * C::kPad + 4 * (sl >> 1)));
#pragma unroll
                                    for (int m = 0; m < MT; ++m) {
                                        const float v =
                                            ((p0[m] + p1[m]) + (q0[m] + q1[m])) + ((r0[m] + r1[m]) + (u0[m] + u1[m]));
                                        acc[i][m] = pr.mode == kSRow ? acc[i][m] + v : fmaf(al, v, acc[i][m]);
                                    }
                                }
                            }
                            __syncwarp();
                            if (lane == 0) mbar_arrive(empty(s));
                            ++k;
                        }
                    }
                }
                if (!ok) break;
                // the K reduction: every warp's partials, summed over the warps in order
#pragma unroll
                for (int i = 0; i < kCSeg; ++i)
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (i < sg.n) sts_f32(red + 4 * (((w * kCSeg + i) * MT + m) * kCRows + r), acc[i][m]);
                if (!(ok = csync())) break;
                if (w < sg.n * MT) {
                    const int i = w / MT, m = w - i * MT;
                    float sum = 0.0f;
#pragma unroll
                    for (int v = 0; v < kSConsumers; ++v) sum += lds_f32(red + 4 * (((v * kCSeg + i) * MT + m) * kCRows + r));
                    const int n = (sg.it + i) * kCRows + r;
                    if (n < pr.N) {
                        if (pr.mode == kSRow) sum *= __ldg(pr.scales + (pr.per_tensor ? 0 : n));
                        if (P.y_bf16)
                            reinterpret_cast<__nv_bfloat16*>(pr.Y)[(int64_t)m * pr.N + n] = __float2bfloat16_rn(sum);
                        else
                            reinterpret_cast<float*>(pr.Y)[(int64_t)m * pr.N + n] = sum;
                    }
                }
                g += sg.n;
            }
            if (!ok) break;
            // arrival: every warp's Y stores of this phase precede its arrival at the consumer
            // barrier (a release at CTA scope), which thread 0's wait acquires, so thread 0's
            // GPU-scope release reduction publishes them all (releases are cumulative); a
            // full fence here cost about 0.4 us per phase
            if (!(ok = csync())) break;
            if (t == 0) red_release_add(P.phase_cnt + ph, 1);
        }
    }
    __syncthreads();
    if (t == 0 && !*abort_flag) {
        // the last CTA to leave zeroes the phase counters for the next launch
        __threadfence();
        if (atomicAdd(P.phase_cnt + P.n_phases, 1) == (int)gridDim.x - 1) {
            for (int ph = 0; ph <= P.n_phases; ++ph) P.phase_cnt[ph] = 0;
            __threadfence();
        }
    }
}

// ---- host side -------------------------------------------------------------------

// Units of W words: K a multiple of 32 W; group scales of 128 or 256 weights
// (whole groups per unit), or row scales.
template <int W>
static bool stream_shape_ok(const ProbShape& s) {
    if (s.N == 0) return false;
    if ((s.N + kSRows - 1) / kSRows > kMaxTickets - kChainCtrs) return false;
    if (s.K % (32 * W) != 0) return false;
    if (s.N * (s.K / 8) >= (int64_t(1) << 32) - 64) return false;  // 32-bit byte offsets into the planes
    if (s.granularity == SHERRY_PER_TENSOR || s.granularity == SHERRY_PER_CHANNEL) return true;
    if (s.granularity != SHERRY_PER_GROUP) return false;
    return s.group == 128 || s.group == 256;
}
template <int W>
static bool stream_eligible_w(const ProbShape& s, int64_t M) {
    return M >= 1 && M <= (W == 16 ? 3 : 4) && stream_shape_ok<W>(s);
}

// one and two tokens: lookup tables on 16-word units (the three- and four-token
// lookup forms serve the chained launches; independent linears of three or more
// tokens go to the tensor-core consumers, which expand each block once)
bool stream_eligible(const ProbShape& s, int64_t M) { return M <= 2 && stream_eligible_w<16>(s, M); }
// three to sixteen tokens: the tensor-core consumers on 16-word units
bool mstream_eligible(const ProbShape& s, int64_t M) { return M >= 3 && M <= 16 && stream_shape_ok<16>(s); }
bool chain_eligible(const ProbShape& s, int64_t M) {
    return M <= 3 ? stream_eligible_w<16>(s, M) : stream_eligible_w<8>(s, M);
}

int64_t stream_tiles(const ProbShape& s) { return (s.N + kSRows - 1) / kSRows; }

// wait budget of the launches (sherry_set_wait_budget)
static std::atomic<long long> g_stream_wait{kSWaitCycles};

long long stream_set_wait_cycles(long long cycles) {
    return g_stream_wait.exchange(cycles > 0 ? cycles : kSWaitCycles);
}

struct SPlan {
    std::vector<SProb> probs;
    std::vector<int> ph_unit, ph_upc;
    int total_units = 0, total_tiles = 0, grid = 0;
    size_t ws_bytes = 0, part_off = 0;
};

// phase_begin: n_phases + 1 problem indices (null: one phase of all problems).
// Independent problems: one CTA per SM at most (the stages fill shared memory)
// and no more CTAs than units; chained phases: one CTA per SM (cooperative).
static SPlan make_splan(const ProbShape* shapes, int count, const int* phase_begin, int n_phases, int64_t M,
                        int sms, int W) {
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
        p.n_sub = (p.words + W - 1) / W;
        p.unit_begin = ub;
        p.tile_begin = tb;
        ub += p.n_rb * p.n_sub;
        tb += p.n_rb;
        pl.probs.push_back(p);
    }
    pl.total_units = ub;
    pl.total_tiles = tb;
    if (phase_begin == nullptr) {
        const int g = std::max(1, std::min(sms, ub));
        const int upc = std::max(1, (ub + g - 1) / g);
        pl.ph_unit = {0, ub};
        pl.ph_upc = {upc};
        pl.grid = std::max(1, (ub + upc - 1) / upc);
    } else {
        pl.grid = std::max(1, sms);
        for (int ph = 0; ph < n_phases; ++ph) {
            const int b = phase_begin[ph] < count ? pl.probs[phase_begin[ph]].unit_begin : ub;
            const int e = phase_begin[ph + 1] < count ? pl.probs[phase_begin[ph + 1]].unit_begin : ub;
            pl.ph_unit.push_back(b);
            pl.ph_upc.push_back(std::max(1, (e - b + pl.grid - 1) / pl.grid));
        }
        pl.ph_unit.push_back(ub);
    }
    pl.part_off = kTicketBytes;
    pl.ws_bytes = kTicketBytes + (size_t)pl.grid * 2 * (size_t)M * kSRows * sizeof(float);
    return pl;
}

size_t stream_workspace_bytes(const ProbShape* shapes, int count, int64_t M, int sms) {
    return make_splan(shapes, count, nullptr, 1, M, sms, 16).ws_bytes;
}

size_t chain_workspace_bytes(const ProbShape* shapes, int count, const int* phase_begin, int n_phases, int64_t M,
                             int sms) {
    if (M <= 2) return kTicketBytes;  // the row-block kernel keeps only its phase counters there
    return make_splan(shapes, count, phase_begin, n_phases, M, sms, M <= 3 ? 16 : 8).ws_bytes;
}

template <int MAXP, int MT, int W>
static int stream_launch_t(SPlan& pl, int y_bf16, void* workspace, bool chain, cudaStream_t stream) {
    static SParams<MAXP> P;
    static std::mutex mu;
    static PerDevice attr;
    std::lock_guard<std::mutex> lk(mu);
    P.wait_cycles = g_stream_wait.load();
    P.count = (int)pl.probs.size();
    P.y_bf16 = y_bf16;
    P.n_phases = (int)pl.ph_upc.size();
    P.ticket = static_cast<int*>(workspace);
    P.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.part_off);
    P.phase_cnt = chain ? static_cast<int*>(workspace) + (kMaxTickets - kChainCtrs) : nullptr;
    for (int i = 0; i < P.count; ++i) P.p[i] = pl.probs[i];
    for (int i = 0; i <= P.n_phases; ++i) P.ph_unit[i] = pl.ph_unit[i];
    for (int i = 0; i < P.n_phases; ++i) P.ph_upc[i] = pl.ph_upc[i];
    int done = 0;
    const int st = per_device(attr, &done, [](int& v) {
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_lut_stream<MAXP, MT, W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               SCfg<MT, W>::kSmem));
        v = 1;
        return SHERRY_OK;
    });
    if (st) return st;
    if (!chain) {
        k_lut_stream<MAXP, MT, W><<<pl.grid, kSThreads, SCfg<MT, W>::kSmem, stream>>>(P);
    } else {
        // every CTA must be resident: the phase barrier waits for all of them
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)pl.grid);
        cfg.blockDim = dim3(kSThreads);
        cfg.dynamicSmemBytes = SCfg<MT, W>::kSmem;
        cfg.stream = stream;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeCooperative;
        at[0].val.cooperative = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        SHERRY_CUDA_CHECK(cudaLaunchKernelEx(&cfg, k_lut_stream<MAXP, MT, W>, P));
    }
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

template <int MT, int W>
static int stream_launch_mt(SPlan& pl, int slots, int y_bf16, void* workspace, bool chain, cudaStream_t stream) {
    if (slots <= 1) return stream_launch_t<1, MT, W>(pl, y_bf16, workspace, chain, stream);
    if (slots <= 16) return stream_launch_t<16, MT, W>(pl, y_bf16, workspace, chain, stream);
    return stream_launch_t<SHERRY_MAX_BATCH, MT, W>(pl, y_bf16, workspace, chain, stream);
}

static void attach(SPlan& pl, const sherry_linear_desc* descs, int count) {
    for (int i = 0; i < count; ++i) {
        SProb& p = pl.probs[i];
        p.X = descs[i].X;
        p.idx = descs[i].idx;
        p.sgn = descs[i].sgn;
        p.scales = descs[i].scales;
        p.Y = descs[i].Y;
    }
}

int stream_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                         void* workspace, int sms, cudaStream_t stream) {
    if (M < 1 || M > 3) return SHERRY_ERR_UNSUPPORTED;
    SPlan pl = make_splan(shapes, count, nullptr, 1, M, sms, 16);
    attach(pl, descs, count);
    if (pl.total_units == 0) return SHERRY_OK;
    switch (M) {
        case 1: return stream_launch_mt<1, 16>(pl, count, y_bf16, workspace, false, stream);
        case 2: return stream_launch_mt<2, 16>(pl, count, y_bf16, workspace, false, stream);
        default: return stream_launch_mt<3, 16>(pl, count, y_bf16, workspace, false, stream);
    }
}

template <int MAXP, int NT>
static int mstream_launch_t(SPlan& pl, int64_t M, int y_bf16, void* workspace, cudaStream_t stream) {
    static SParams<MAXP> P;
    static std::mutex mu;
    static PerDevice attr;
    std::lock_guard<std::mutex> lk(mu);
    P.wait_cycles = g_stream_wait.load();
    P.count = (int)pl.probs.size();
    P.y_bf16 = y_bf16;
    P.n_phases = 1;
    P.ticket = static_cast<int*>(workspace);
    P.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.part_off);
    P.phase_cnt = nullptr;
    for (int i = 0; i < P.count; ++i) P.p[i] = pl.probs[i];
    P.ph_unit[0] = pl.ph_unit[0];
    P.ph_unit[1] = pl.ph_unit[1];
    P.ph_upc[0] = pl.ph_upc[0];
    int done = 0;
    const int st = per_device(attr, &done, [](int& v) {
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_mma_stream<MAXP, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               MCfg<NT>::kSmem));
        v = 1;
        return SHERRY_OK;
    });
    if (st) return st;
    k_mma_stream<MAXP, NT><<<pl.grid, kSThreads, MCfg<NT>::kSmem, stream>>>(P, (int)M);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

template <int NT>
static int mstream_launch_nt(SPlan& pl, int count, int64_t M, int y_bf16, void* workspace, cudaStream_t stream) {
    if (count <= 1) return mstream_launch_t<1, NT>(pl, M, y_bf16, workspace, stream);
    if (count <= 16) return mstream_launch_t<16, NT>(pl, M, y_bf16, workspace, stream);
    return mstream_launch_t<SHERRY_MAX_BATCH, NT>(pl, M, y_bf16, workspace, stream);
}

int mstream_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                          void* workspace, int sms, cudaStream_t stream) {
    if (M < 1 || M > 16) return SHERRY_ERR_UNSUPPORTED;
    SPlan pl = make_splan(shapes, count, nullptr, 1, M, sms, 16);
    attach(pl, descs, count);
    if (pl.total_units == 0) return SHERRY_OK;
    return M <= 8 ? mstream_launch_nt<8>(pl, count, M, y_bf16, workspace, stream)
                  : mstream_launch_nt<16>(pl, count, M, y_bf16, workspace, stream);
}

bool chain_launch_ok(const ProbShape* shapes, int count, int n_phases, int64_t M) {
    if (M < 1 || M > 4 || n_phases > kSMaxPhases || n_phases > SHERRY_MAX_BATCH || count > SHERRY_MAX_BATCH)
        return false;
    int64_t tiles = 0;
    for (int i = 0; i < count; ++i) {
        if (!chain_eligible(shapes[i], M)) return false;
        tiles += stream_tiles(shapes[i]);
    }
    return tiles <= kMaxTickets - kChainCtrs;
}

// Chains of one or two tokens run on the row-block kernel (k_lut_rows): every linear's
// items are 32 rows over all of K, so no row block is split over CTAs.  Shapes are
// those of the streaming kernel (K a multiple of 512: whole 16-byte slices per row
// and 16-byte aligned row starts in every plane).
template <int MAXP, int MT>
static int rows_launch_t(const ProbShape* shapes, const sherry_linear_desc* descs, int count, const int* phase_begin,
                         int n_phases, int y_bf16, void* workspace, int sms, cudaStream_t stream) {
    static CParams<MAXP> P;
    static std::mutex mu;
    static PerDevice attr;
    std::lock_guard<std::mutex> lk(mu);
    P.wait_cycles = g_stream_wait.load();
    P.count = count;
    P.y_bf16 = y_bf16;
    P.n_phases = n_phases;
    P.phase_cnt = static_cast<int*>(workspace) + (kMaxTickets - kChainCtrs);
    int items = 0;
    for (int i = 0; i < count; ++i) {
        const ProbShape& sh = shapes[i];
        CProb c{};
        c.X = descs[i].X;
        c.idx = descs[i].idx;
        c.sgn = descs[i].sgn;
        c.scales = descs[i].scales;
        c.Y = descs[i].Y;
        c.N = (int)sh.N;
        c.K = (int)sh.K;
        c.spr = sh.granularity == SHERRY_PER_GROUP ? (int)(sh.K / sh.group) : 0;
        c.mode = sh.granularity != SHERRY_PER_GROUP ? kSRow : (sh.group == 128 ? kSG128 : kSG256);
        c.per_tensor = sh.granularity == SHERRY_PER_TENSOR;
        c.n_items = (int)((sh.N + kCRows - 1) / kCRows);
        c.item_begin = items;
        items += c.n_items;
        P.p[i] = c;
    }
    for (int ph = 0; ph <= n_phases; ++ph) {
        P.ph_prob[ph] = phase_begin[ph];
        P.ph_item[ph] = phase_begin[ph] < count ? P.p[phase_begin[ph]].item_begin : items;
    }
    int done = 0;
    const int st = per_device(attr, &done, [](int& v) {
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_lut_rows<MAXP, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               CCfg<MT>::kSmem));
        v = 1;
        return SHERRY_OK;
    });
    if (st) return st;
    // every CTA must be resident: the phase barrier waits for all of them
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::max(1, sms));
    cfg.blockDim = dim3(kSThreads);
    cfg.dynamicSmemBytes = CCfg<MT>::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    SHERRY_CUDA_CHECK(cudaLaunchKernelEx(&cfg, k_lut_rows<MAXP, MT>, P));
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

template <int MT>
static int rows_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, const int* phase_begin,
                       int n_phases, int y_bf16, void* workspace, int sms, cudaStream_t stream) {
    const int slots = std::max(count, n_phases);
    if (slots <= 1) return rows_launch_t<1, MT>(shapes, descs, count, phase_begin, n_phases, y_bf16, workspace, sms, stream);
    if (slots <= 16)
        return rows_launch_t<16, MT>(shapes, descs, count, phase_begin, n_phases, y_bf16, workspace, sms, stream);
    return rows_launch_t<SHERRY_MAX_BATCH, MT>(shapes, descs, count, phase_begin, n_phases, y_bf16, workspace, sms,
                                               stream);
}

int chain_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, const int* phase_begin,
                        int n_phases, int64_t M, int y_bf16, void* workspace, int sms, cudaStream_t stream) {
    if (!chain_launch_ok(shapes, count, n_phases, M)) return SHERRY_ERR_UNSUPPORTED;
    if (M == 1) return rows_launch<1>(shapes, descs, count, phase_begin, n_phases, y_bf16, workspace, sms, stream);
    if (M == 2) return rows_launch<2>(shapes, descs, count, phase_begin, n_phases, y_bf16, workspace, sms, stream);
    SPlan pl = make_splan(shapes, count, phase_begin, n_phases, M, sms, M <= 3 ? 16 : 8);
    attach(pl, descs, count);
    // the kernel's phase table has one slot per problem slot of its instantiation
    const int slots = std::max(count, n_phases);
    switch (M) {
        case 1: return stream_launch_mt<1, 16>(pl, slots, y_bf16, workspace, true, stream);
        case 2: return stream_launch_mt<2, 16>(pl, slots, y_bf16, workspace, true, stream);
        case 3: return stream_launch_mt<3, 16>(pl, slots, y_bf16, workspace, true, stream);
        default: return stream_launch_mt<4, 8>(pl, slots, y_bf16, workspace, true, stream);
    }
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
