// gemv_tc.cu -- packed 3:4 ternary linear for a few tokens (9 <= M <= 32) on the
// tensor cores, Y = X (T alpha)^T ("Sherry: Hardware-Efficient 1.25-Bit Ternary
// Quantization via Fine-grained Sparsification", digest: Y = X T alpha).
//
// With a handful of tokens the lookup-table decode does one table lookup per
// block and token; here every weight is expanded once to bf16 {-1, 0, +1} (one
// pattern-table lookup per block, whatever M is) and multiplied on the tensor
// cores with all tokens at once (MMA N = 16 or 32 token columns).  Like the
// one-token kernel it streams the packed planes from HBM once, for any number
// of independent linears in one launch.
//
// Work unit: one linear's 128 weight rows x all of K.  Units are dealt to one
// persistent CTA per SM round-robin; K advances in chunks of 256 weights (four
// 64-weight MMA steps).  Per CTA (25 warps):
//   warps 0-3    epilogue (TMEM lane quarter = warp % 4): promote each scale
//                group's accumulator with alpha in fp32 registers, write Y
//   warps 4-19   decode, four groups of four warps: group g expands step g of
//                every chunk, one TMEM lane (= weight row) per thread, 16
//                pattern lookups per thread -> tcgen05.st (operand A in TMEM).
//                Four groups keep four independent decode chains in flight.
//   warps 20-22  producers: cp.async of each chunk -- the packed words (stored
//                step-major so a group's reads are conflict-free), the sign
//                bytes, and the X chunk laid out as the MMA's SWIZZLE_128B
//                K-major B operand (rows >= M are zeroed once, never copied);
//                completion is signalled on an mbarrier (cp.async.mbarrier.arrive)
//   warps 23-24  TMEM allocation (warp 23); one thread of each issues the
//                tcgen05.mma sub-steps kk = me, me + 2 of every step (A from TMEM,
//                B from shared memory) into its own column slice of the
//                accumulator; the epilogue adds the two slices
// Every mbarrier wait is bounded.
#include "common.cuh"
#include "lut.cuh"

#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <vector>

namespace sherry {

constexpr int kTDecGroups = 4;                      // decode groups (one per step of a chunk)
constexpr int kTProdWarps = 2;                      // producer warps
constexpr int kTMmaWarps = 2;                       // MMA-issuing warps (one thread each)
constexpr int kTThreads = 32 * (4 + 4 * kTDecGroups + kTProdWarps + kTMmaWarps);  // 25 warps
constexpr int kTProdWarp = 4 + 4 * kTDecGroups;     // first producer warp (20)
constexpr int kTMmaWarp = kTProdWarp + kTProdWarps; // first MMA warp (23)
constexpr int kTRows = 128;               // weight rows per unit (MMA M, TMEM lanes)
constexpr int kTStepK = 64;               // K per MMA step (one 128-byte swizzle atom of bf16)
constexpr int kTChunkSteps = 4;           // steps per staged chunk (256 weights)
constexpr int kTChunkK = kTStepK * kTChunkSteps;
constexpr int kTChunks = 6;               // staged chunks in flight
constexpr int kTAcc = 4;                  // group accumulators, each split in kTMmaWarps column slices
constexpr int kTTmemCols = 512;           // accumulators first, then the A stages
constexpr int kTAParMax = 3;              // A buffers per decode group, at most
constexpr int kTIdxBytes = kTRows * kTChunkSteps * 8;    // 4 KB: [step][row] 8 bytes (2 words)
constexpr int kTSgnBytes = kTRows * kTChunkSteps * 2;    // 1 KB: [row] 8 sign bytes
constexpr long long kTWaitCycles = 4000000000LL;
// below this many tokens the warp-level MMA kernel is faster (measured on the 3B
// decode stack: M = 8: 0.566 vs 0.620 ms; M = 16: 0.760 vs 0.634 ms)
constexpr int kSkinnyMinM = 9;
static_assert(kTDecGroups == kTChunkSteps, "one decode group per chunk step");
static_assert(kTAParMax < kTChunks, "an A buffer's release is still tracked by its chunk slot");

struct TProb {
    const uint16_t* X;
    const uint32_t* idx;
    const uint8_t* sgn;
    const float* scales;
    void* Y;
    int N, K, words;
    int row_scale, per_tensor, spr, group_steps;
    int unit_begin, n_rt;
};

template <int MAXP>
struct TParams {
    int count, M, y_bf16, total_units;
    TProb p[MAXP];
};

// bounded-wait timeouts of this file's kernel (read and cleared by sherry_device_status)
__device__ int g_skinny_status = 0;

namespace {

__device__ __forceinline__ void t_mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void t_mbar_arrive(uint32_t bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool t_mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool t_mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (t_mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (t_mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kTWaitCycles) {
            *abort_flag = 1;
            atomicExch(&g_skinny_status, SHERRY_ERR_TIMEOUT);
            return false;
        }
    }
}
// Bounded wait used on the way out (normal finish or abort): it ignores the
// abort flag so that the MMAs this CTA committed complete before TMEM is freed.
__device__ __forceinline__ void t_mbar_drain(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!t_mbar_try(bar, parity)) {
        if (clock64() - t0 > kTWaitCycles) {
            atomicExch(&g_skinny_status, SHERRY_ERR_TIMEOUT);
            return;
        }
    }
}
__device__ __forceinline__ void t_cp16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void t_cp8(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(valid ? 8 : 0)
                 : "memory");
}
// the mbarrier receives one arrival when all of this thread's prior cp.async complete
__device__ __forceinline__ void t_cp_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void t_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void t_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ uint64_t t_smem_desc(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3fff);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

template <int BN>
struct TIdesc {
    static constexpr uint32_t v =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kTRows >> 4) << 24);
};

__device__ __forceinline__ void t_mma(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void t_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

}  // namespace

#define SHERRY_T_ST32(taddr, v)                                                                                  \
    asm volatile(                                                                                                \
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16," \
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),                        \
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),      \
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),          \
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),         \
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])                      \
        : "memory")

#define SHERRY_T_LD16(taddr, v)                                                                          \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
                 "%15}, [%16];"                                                                          \
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),    \
                   "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), \
                   "=r"(v[14]), "=r"(v[15])                                                               \
                 : "r"(taddr))

// unit u -> (problem, row tile).  A CTA visits its units in increasing order, so
// the problem index only moves forward: `p` is the caller's cursor (start at 0).
template <int MAXP>
__device__ __forceinline__ void t_locate(const TParams<MAXP>& P, int u, int& p, int& rt) {
    while (p + 1 < P.count && P.p[p + 1].unit_begin <= u) ++p;
    rt = u - P.p[p].unit_begin;
}

template <int BN, int MAXP>
__global__ void __launch_bounds__(kTThreads, 1) k_skinny(const __grid_constant__ TParams<MAXP> P) {
    constexpr int kXStep = BN * 128;                 // X bytes per 64-K step (BN rows x 128 B)
    constexpr int kXBytes = kXStep * kTChunkSteps;   // per chunk
    constexpr uint32_t kIdesc = TIdesc<BN>::v;
    constexpr int kAccCols = kTMmaWarps * BN;        // TMEM columns per accumulator
    constexpr int kAcolT = kTAcc * kAccCols;         // first A column
    // A buffers per decode group: as many as TMEM holds (3 for 16 token columns, 2 for 32);
    // A stage (group g, buffer h) at column kAcolT + 32 (kAPar g + h)
    constexpr int kAPar0 = (kTTmemCols - kAcolT) / (32 * kTDecGroups);
    constexpr int kAPar = kAPar0 < kTAParMax ? kAPar0 : kTAParMax;
    static_assert(BN % 16 == 0 && kAPar >= 2, "TMEM plan");
    extern __shared__ __align__(1024) unsigned char tsm[];
    __shared__ uint64_t bars[2 * kTChunks + kTAParMax + 2 * kTAcc + 1];
    __shared__ uint32_t tmem_s;
    __shared__ volatile int abort_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t base = (smem_u32(tsm) + 1023u) & ~1023u;  // X stages first (1024-aligned)
    auto xst = [&](int c) { return base + (uint32_t)(c * kXBytes); };
    const uint32_t pbase = base + (uint32_t)(kTChunks * kXBytes);
    auto ist = [&](int c) { return pbase + (uint32_t)(c * (kTIdxBytes + kTSgnBytes)); };
    const uint32_t table = pbase + (uint32_t)(kTChunks * (kTIdxBytes + kTSgnBytes));  // 256-aligned
    const uint32_t bar0 = smem_u32(&bars[0]);
    auto full_c = [&](int c) { return bar0 + 8u * c; };
    auto empty_c = [&](int c) { return bar0 + 8u * (kTChunks + c); };
    auto full_a = [&](int h) { return bar0 + 8u * (2 * kTChunks + h); };  // A buffer h of every group written
    auto acc_full = [&](int b) { return bar0 + 8u * (2 * kTChunks + kTAParMax + b); };
    auto acc_empty = [&](int b) { return bar0 + 8u * (2 * kTChunks + kTAParMax + kTAcc + b); };
    const uint32_t drain = bar0 + 8u * (2 * kTChunks + kTAParMax + 2 * kTAcc);  // MMA threads' last commits
    const int M = P.M;

    if (threadIdx.x == 0) {
        abort_s = 0;
        for (int c = 0; c < kTChunks; ++c) {
            t_mbar_init(full_c(c), 32 * kTProdWarps);         // the producer warps' cp.async arrivals
            // the MMA commit (X and the chunk's A stages read) + every decode thread (words read)
            t_mbar_init(empty_c(c), kTMmaWarps + 128 * kTDecGroups);
        }
        for (int h = 0; h < kAPar; ++h) t_mbar_init(full_a(h), 128 * kTDecGroups);
        for (int b = 0; b < kTAcc; ++b) {
            t_mbar_init(acc_full(b), kTMmaWarps);
            t_mbar_init(acc_empty(b), 128);
        }
        t_mbar_init(drain, kTMmaWarps);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (threadIdx.x < 32) {
        const uint32_t e = threadIdx.x;
        const uint2 pat = decode_block_bf16(e & 15u, e >> 4);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(table + 4u * e), "r"(pat.x) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(table + 128u + 4u * e), "r"(pat.y) : "memory");
    }
    // token rows M..BN-1 of every X stage stay zero for the whole launch
    for (int q = threadIdx.x; q < kTChunks * kTChunkSteps * (BN - M) * 8; q += kTThreads) {
        const int cq = q & 7, rr = q >> 3;
        const int r = M + rr % (BN - M), cs = rr / (BN - M);
        const uint32_t a = xst(cs / kTChunkSteps) + (uint32_t)((cs % kTChunkSteps) * kXStep + (r >> 3) * 1024 +
                                                               (r & 7) * 128 + (cq << 4));
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == kTMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_s)),
                     "r"(kTTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    t_fence_before();
    __syncthreads();
    t_fence_after();
    const uint32_t tmem = tmem_s;

    if (warp >= kTProdWarp && warp < kTProdWarp + kTProdWarps) {
        // ---------------- producers: copy job j of a chunk goes to warp j % kTProdWarps ----------------
        const int pw = warp - kTProdWarp;
        int cc = 0;  // chunks produced (all units)
        int p = 0;   // problem cursor
        bool ok = true;
        for (int u = blockIdx.x; u < P.total_units && ok; u += gridDim.x) {
            int rt;
            t_locate(P, u, p, rt);
            const TProb& pr_ = P.p[p];
            const uint16_t* const pr_X = pr_.X;
            const uint32_t* const pr_idx = pr_.idx;
            const uint8_t* const pr_sgn = pr_.sgn;
            const int pr_N = pr_.N, pr_K = pr_.K, pr_words = pr_.words;
            const int row0 = rt * kTRows;
            const int nchunks = pr_K / kTChunkK;
            for (int ch = 0; ch < nchunks; ++ch, ++cc) {
                const int c = cc % kTChunks;
                if (!t_mbar_wait(empty_c(c), (uint32_t)(((cc / kTChunks) & 1) ^ 1), &abort_s)) {
                    ok = false;
                    break;
                }
                const int w0 = ch * kTChunkSteps * 2;  // first packed word of the chunk
                // packed words: 128 rows x 4 steps x 8 B, stored [step][row]
#pragma unroll
                for (int i = pw; i < 16; i += kTProdWarps) {
                    const int q = lane + 32 * i;
                    const int r = q >> 2, g = q & 3;
                    const int row = row0 + r;
                    const bool v = row < pr_N;
                    t_cp8(ist(c) + g * (kTRows * 8) + r * 8,
                          v ? (const void*)(pr_idx + (int64_t)row * pr_words + w0 + 2 * g) : (const void*)pr_idx, v);
                }
                // sign bytes: 128 rows x 8 B
#pragma unroll
                for (int i = pw; i < 4; i += kTProdWarps) {
                    const int r = lane + 32 * i;
                    const int row = row0 + r;
                    const bool v = row < pr_N;
                    t_cp8(ist(c) + kTIdxBytes + r * 8,
                          v ? (const void*)(pr_sgn + (int64_t)row * pr_words + w0) : (const void*)pr_sgn, v);
                }
                // X chunk, token rows < M: 4 steps x 8 pieces of 16 B per row, SWIZZLE_128B K-major
                for (int r = pw; r < M; r += kTProdWarps) {
                    const int st = lane >> 3, cq = lane & 7;
                    const int kk = ch * kTChunkK + st * kTStepK + cq * 8;
                    t_cp16(xst(c) + st * kXStep + (r >> 3) * 1024 + (r & 7) * 128 + ((cq ^ (r & 7)) << 4),
                           pr_X + (int64_t)r * pr_K + kk, true);
                }
                t_cp_arrive(full_c(c));
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp >= 4 && warp < kTProdWarp) {
        // ---------------- decode: group g expands step g of every chunk ----------------
        const int g = (warp - 4) >> 2, q = warp & 3, i = q * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)kAcolT;
        int cc = 0, p = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < P.total_units && ok; u += gridDim.x) {
            int rt;
            t_locate(P, u, p, rt);
            const int nchunks = P.p[p].K / kTChunkK;
            for (int ch = 0; ch < nchunks; ++ch, ++cc) {
                const int c = cc % kTChunks;
                if (!t_mbar_wait(full_c(c), (uint32_t)((cc / kTChunks) & 1), &abort_s)) {
                    ok = false;
                    break;
                }
                uint32_t w_lo, w_hi, sg;
                asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                             : "=r"(w_lo), "=r"(w_hi)
                             : "r"(ist(c) + g * (kTRows * 8) + i * 8));
                asm volatile("ld.shared.u16 %0, [%1];" : "=r"(sg) : "r"(ist(c) + kTIdxBytes + i * 8 + 2 * g));
                t_mbar_arrive(empty_c(c));  // this thread has its words
                uint32_t v[32];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t wd = h ? w_hi : w_lo;
                    const uint32_t sb = (sg >> (8 * h)) & 0xffu;
                    const uint32_t ev = ((wd << 2) & 0x3c3c3c3cu) | (((sb & 0x55u) * 0x01041040u) & 0x40404040u);
                    const uint32_t od = ((wd >> 2) & 0x3c3c3c3cu) | (((sb & 0xaau) * 0x00820820u) & 0x40404040u);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t a = __byte_perm((j & 1) ? od : ev, table, (uint32_t)(j >> 1) | 0x7650u);
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v[16 * h + 2 * j]) : "r"(a));
                        asm volatile("ld.shared.u32 %0, [%1+128];" : "=r"(v[16 * h + 2 * j + 1]) : "r"(a));
                    }
                }
                // stage (g, cc % kAPar) was last read by the MMAs of chunk cc - kAPar, whose
                // completion the MMA threads commit to that chunk's slot barrier
                const int h = cc % kAPar;
                const int s = kAPar * g + h;
                if (cc >= kAPar) {
                    const int c2 = (cc - kAPar) % kTChunks;
                    if (!t_mbar_wait(empty_c(c2), (uint32_t)(((cc - kAPar) / kTChunks) & 1), &abort_s)) {
                        ok = false;
                        break;
                    }
                }
                t_fence_after();
                SHERRY_T_ST32(t_lane + (uint32_t)(s * 32), v);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                t_fence_before();
                t_mbar_arrive(full_a(h));
            }
        }
    } else if (warp >= kTMmaWarp) {
        // ---------------- MMA issuers: warp kTMmaWarp + me issues sub-steps kk of every step
        // with kk % kTMmaWarps == me into its own column slice of the accumulator ----------------
        const int me = warp - kTMmaWarp;
        // One wait per chunk (all four A stages written; the decode threads had
        // waited for the chunk's X, so it has landed too), 16 MMAs, one commit
        // per chunk; group bookkeeping by counters only.
        if (lane == 0) {
            int cc = 0, c = 0, p = 0;
            uint32_t cph = 0;           // phase parity of slot c
            int b = 0;                  // accumulator
            uint32_t bph = 0;           // phase parity of accumulator b's use
            bool ok = true;
            for (int u = blockIdx.x; u < P.total_units && ok; u += gridDim.x) {
                int rt;
                t_locate(P, u, p, rt);
                const int nchunks = P.p[p].K / kTChunkK, gs = P.p[p].group_steps;
                int gstep = 0;          // steps done in the current group
                for (int ch = 0; ch < nchunks; ++ch, ++cc) {
                    const int h = cc % kAPar;
                    if (!t_mbar_wait(full_a(h), (uint32_t)((cc / kAPar) & 1), &abort_s)) { ok = false; break; }
                    // X arrived through cp.async (generic proxy); the MMA reads it through the async proxy
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    t_fence_after();
                    const uint64_t db0 = t_smem_desc(xst(c));
                    const uint32_t ta0 = tmem + (uint32_t)(kAcolT + h * 32);
#pragma unroll
                    for (int st = 0; st < kTChunkSteps; ++st) {
                        if (gstep == 0) {
                            if (!t_mbar_wait(acc_empty(b), bph ^ 1u, &abort_s)) { ok = false; break; }
                            t_fence_after();
                        }
                        const uint32_t td = tmem + (uint32_t)(b * kAccCols + me * BN);
                        const uint32_t ta = ta0 + (uint32_t)(st * kAPar * 32);
                        const uint64_t db = db0 + (uint64_t)((st * kXStep) >> 4);
#pragma unroll
                        for (int kk = me; kk < kTStepK / 16; kk += kTMmaWarps)
                            t_mma(td, ta + (uint32_t)(8 * kk), db + (uint64_t)(2 * kk), kIdesc,
                                  (gstep == 0 && kk == me) ? 0u : 1u);
                        if (++gstep == gs) {
                            t_commit(acc_full(b));
                            gstep = 0;
                            if (++b == kTAcc) { b = 0; bph ^= 1u; }
                        }
                    }
                    if (!ok) break;
                    t_commit(empty_c(c));
                    if (++c == kTChunks) { c = 0; cph ^= 1u; }
                }
            }
            (void)cph;
            // the MMAs of both issuers complete before TMEM is freed (after an abort
            // no epilogue has waited for them)
            t_commit(drain);
            t_mbar_drain(drain, 0u);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: unit row 32*warp + lane per thread ----------------
        int gc = 0, p = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < P.total_units && ok; u += gridDim.x) {
            int rt;
            t_locate(P, u, p, rt);
            const TProb& pr_ = P.p[p];
            const float* const pr_scales = pr_.scales;
            void* const pr_Y = pr_.Y;
            const int pr_N = pr_.N, pr_spr = pr_.spr;
            const int row_scale = pr_.row_scale, per_tensor = pr_.per_tensor;
            const int n = rt * kTRows + warp * 32 + lane;
            const bool row_ok = n < pr_N;
            const int ngroups = (pr_.K / kTStepK) / pr_.group_steps;
            const float* srow = pr_scales + (int64_t)(row_ok ? n : 0) * pr_spr;
            // group scales are loaded two groups ahead of their use
            const bool gsc = !row_scale && row_ok;
            float a_next = gsc ? __ldg(srow) : 1.0f;
            float a_next2 = (gsc && ngroups > 1) ? __ldg(srow + 1) : 1.0f;
            float acc[BN];
#pragma unroll
            for (int j = 0; j < BN; ++j) acc[j] = 0.0f;
            for (int gi = 0; gi < ngroups; ++gi, ++gc) {
                const float a = a_next;
                a_next = a_next2;
                a_next2 = (gsc && gi + 2 < ngroups) ? __ldg(srow + gi + 2) : 1.0f;
                const int b = gc % kTAcc;
                ok = t_mbar_wait(acc_full(b), (uint32_t)((gc / kTAcc) & 1), &abort_s);
                if (!ok) break;
                t_fence_after();
                const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(b * kAccCols);
                // 16 token columns at a time: the slices' partial sums, added in a fixed order
#pragma unroll
                for (int c = 0; c < BN / 16; ++c) {
                    uint32_t v[16 * kTMmaWarps];
#pragma unroll
                    for (int m = 0; m < kTMmaWarps; ++m) SHERRY_T_LD16(t_row + m * BN + 16 * c, (v + 16 * m));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float g = __uint_as_float(v[j]);
#pragma unroll
                        for (int m = 1; m < kTMmaWarps; ++m) g += __uint_as_float(v[16 * m + j]);
                        acc[16 * c + j] = fmaf(a, g, acc[16 * c + j]);
                    }
                }
                t_fence_before();
                t_mbar_arrive(acc_empty(b));
            }
            if (ok && row_ok) {
                const float a = row_scale ? __ldg(pr_scales + (per_tensor ? 0 : n)) : 1.0f;
#pragma unroll
                for (int j = 0; j < BN; ++j) {
                    if (j < M) {
                        const float y = acc[j] * a;
                        if (P.y_bf16)
                            reinterpret_cast<__nv_bfloat16*>(pr_Y)[(int64_t)j * pr_N + n] = __float2bfloat16_rn(y);
                        else
                            reinterpret_cast<float*>(pr_Y)[(int64_t)j * pr_N + n] = y;
                    }
                }
            }
        }
    }

    t_fence_before();
    __syncthreads();
    if (warp == kTMmaWarp) {
        t_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTTmemCols));
    }
}

}  // namespace sherry

// ---- host side -------------------------------------------------------------------

namespace sherry {

bool skinny_eligible(const ProbShape& s, int64_t M) {
    if (M < kSkinnyMinM || M > 32 || s.N == 0) return false;
    if (s.K % kTChunkK != 0) return false;
    if (s.granularity == SHERRY_PER_GROUP && s.group % kTStepK != 0) return false;
    return true;
}

template <int BN>
static constexpr int skinny_smem() {
    return kTChunks * (BN * 128 * kTChunkSteps + kTIdxBytes + kTSgnBytes) + 256 + 1024;  // + table + alignment
}

template <int BN, int MAXP>
static int skinny_launch_t(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M,
                           int y_bf16, int sms, cudaStream_t stream) {
    static TParams<MAXP> P;
    static std::mutex mu;
    static PerDevice attr;
    std::lock_guard<std::mutex> lk(mu);
    P.count = count;
    P.M = (int)M;
    P.y_bf16 = y_bf16;
    int ub = 0;
    for (int i = 0; i < count; ++i) {
        const ProbShape& s = shapes[i];
        TProb& p = P.p[i];
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
        p.group_steps = s.granularity == SHERRY_PER_GROUP ? s.group / kTStepK : (int)(s.K / kTStepK);
        p.n_rt = (int)((s.N + kTRows - 1) / kTRows);
        p.unit_begin = ub;
        ub += p.n_rt;
    }
    P.total_units = ub;
    if (ub == 0) return SHERRY_OK;
    constexpr int smem = skinny_smem<BN>();
    int done = 0;
    const int st = per_device(attr, &done, [](int& v) {
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_skinny<BN, MAXP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        v = 1;
        return SHERRY_OK;
    });
    if (st) return st;
    const int grid = ub < sms ? ub : sms;
    k_skinny<BN, MAXP><<<grid, kTThreads, smem, stream>>>(P);
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

template <int BN>
static int skinny_launch_n(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M,
                           int y_bf16, int sms, cudaStream_t stream) {
    if (count <= 1) return skinny_launch_t<BN, 1>(shapes, descs, count, M, y_bf16, sms, stream);
    if (count <= 16) return skinny_launch_t<BN, 16>(shapes, descs, count, M, y_bf16, sms, stream);
    return skinny_launch_t<BN, SHERRY_MAX_BATCH>(shapes, descs, count, M, y_bf16, sms, stream);
}

int skinny_status_take() {
    int v = 0;
    SHERRY_CUDA_CHECK(cudaMemcpyFromSymbol(&v, g_skinny_status, sizeof(int)));
    if (v) {
        const int zero = 0;
        SHERRY_CUDA_CHECK(cudaMemcpyToSymbol(g_skinny_status, &zero, sizeof(int)));
    }
    return v;
}

int skinny_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                         int sms, cudaStream_t stream) {
    if (M <= 16) return skinny_launch_n<16>(shapes, descs, count, M, y_bf16, sms, stream);
    return skinny_launch_n<32>(shapes, descs, count, M, y_bf16, sms, stream);
}

}  // namespace sherry
