// prefill.cu -- packed 3:4 ternary linear for many tokens on the 5th-generation
// tensor cores (tcgen05 + TMEM), Y = X (T alpha)^T ("Sherry: Hardware-Efficient
// 1.25-Bit Ternary Quantization via Fine-grained Sparsification", digest: Y = X
// T alpha; "Sherry, Tequila and Fairies in Python" section 1.1: F.linear).
//
// With many tokens the layer is a dense contraction, so the packed weights are
// expanded to bf16 {-1, 0, +1} and multiplied on the tensor cores; alpha cannot
// be folded into the bf16 weights without losing precision, so each K-group is
// accumulated separately in TMEM and promoted into fp32 registers with alpha
// (per-row scales: once at the end).
//
// CTA tile: 128 weight rows (MMA M, TMEM lanes) x 128 tokens (MMA N); K runs in
// chunks of 256 (four 64-wide MMA steps).  The expanded weights (MMA operand A)
// never touch shared memory: decode threads own one TMEM lane (= weight row)
// each and write their row's 64 bf16 of a step into TMEM with tcgen05.st; only
// the X tiles (operand B) come through shared memory, by TMA (no multicast).
// Synchronisation is per chunk: the MMA thread waits once for the chunk's four A
// stages and once for its X, issues the 16 MMAs, and commits once; that commit
// frees both the X slot and the chunk's A buffer.
//   warps 0..E-1 epilogue (E = 16 for group scales and K <= 4096, else 8): wait for one of two
//                finished group accumulators, tcgen05.ld its share of the tokens
//                (128 / (E / 4) each), acc[token] += alpha(row, group) * D, write
//                Y (row per thread)
//   next 8 warps decode, two groups of four warps: group g expands steps 2g and
//                2g + 1 of every chunk, one pattern-table lookup per block of 4
//                weights; packed words come straight from global memory through
//                a per-thread prefetch ring
//   next warp    TMA: the chunk's four X tiles [128 tokens x 64 K], SWIZZLE_128B
//   last warp    TMEM allocation; one elected thread issues tcgen05.mma
#include "common.cuh"
#include "lut.cuh"

#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

namespace sherry {

constexpr int kPDecGroups = 2;   // decode groups (two MMA steps of every chunk each)
// epilogue warps EPI (8 or 16; a template parameter of the kernel), then the decode
// warps, the TMA warp and the MMA warp
template <int EPI>
struct PRoles {
    static constexpr int kThreads = 32 * (EPI + 4 * kPDecGroups + 2);
    static constexpr int kTmaWarp = EPI + 4 * kPDecGroups;
    static constexpr int kMmaWarp = kTmaWarp + 1;
};
constexpr int kPBM = 128;     // weight rows per tile
constexpr int kPBN = 128;     // tokens per tile
constexpr int kPBK = 64;      // K per MMA step
constexpr int kPChunkSteps = 4;                  // steps per chunk
constexpr int kPStepB = kPBN * kPBK * 2;         // 16 KB of X per step
constexpr int kPXSlots = 3;                      // X chunks in flight
constexpr int kPABuf = 2;                        // A buffers (chunks) in TMEM
constexpr int kPRing = 2;                        // chunks of packed words in flight per decode thread
constexpr int kPArnSteps = 2, kPArnSlots = 3;    // Arenas: steps per chunk, slots (X and W tiles)
constexpr int kPXBytes = kPXSlots * kPChunkSteps * kPStepB > kPArnSlots * 2 * kPArnSteps * kPStepB
                             ? kPXSlots * kPChunkSteps * kPStepB
                             : kPArnSlots * 2 * kPArnSteps * kPStepB;  // the slots of either form
constexpr int kPTable = 256;                     // 32 weight patterns: low words (128 B), then high words
constexpr int kPSmem = kPXBytes + kPTable + 1024;
constexpr int kPAcc = 2;                         // group accumulators in flight
constexpr int kPTmemCols = 512;                  // 2 x 128 accumulator columns + the A buffers
constexpr int kPAcol = kPAcc * kPBN;             // first TMEM column of the A stages (256)
constexpr int kPAcols = kPBK / 2;                // 32 columns (64 bf16) per A stage
constexpr long long kPWaitCycles = 4000000000LL;  // ~2 s at 2 GHz
constexpr int kPMaxSlots = kPXSlots > kPArnSlots ? kPXSlots : kPArnSlots;
constexpr int kPMaxABuf = kPABuf > 2 ? kPABuf : 2;
static_assert(kPAcol + kPABuf * kPChunkSteps * kPAcols <= kPTmemCols, "TMEM plan");
static_assert(kPXSlots >= kPABuf + 1, "the decode's A-buffer wait reads the slot barrier of chunk cc - kPABuf");

__device__ int g_device_status = 0;

struct PParams {
    const uint32_t* idx;
    const uint8_t* sgn;
    const float* scales;
    void* Y;
    int M, N, K, words;
    int y_bf16;
    int row_scale, per_tensor, spr;
    int group_steps;  // K-steps per scale group (per-row: all of K)
    float lambda;     // Arenas: weight of the dense product
};

// ---- PTX wrappers -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
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
// bounded wait: false if it gave up (or another thread of the CTA did)
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kPWaitCycles) {
            *abort_flag = 1;
            atomicExch(&g_device_status, SHERRY_ERR_TIMEOUT);
            return false;
        }
    }
}
// Bounded wait used on the way out of the kernel, after a normal finish or an
// abort: it ignores the abort flag, so that the CTA's own asynchronous work (its
// committed MMAs, its TMA loads in flight) lands before TMEM is freed and the
// CTA's shared memory is released.  On timeout it records the error and returns.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try(bar, parity)) {
        if (clock64() - t0 > kPWaitCycles) {
            atomicExch(&g_device_status, SHERRY_ERR_TIMEOUT);
            return;
        }
    }
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// K-major, 128-byte swizzled operand: 8-row atoms of 1024 bytes
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3fff);        // start address
    d |= (uint64_t)1 << 16;                       // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;             // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                       // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                       // SWIZZLE_128B
    return d;
}

// bf16 x bf16 -> fp32, both K-major, M = 128, N = 128
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kPBN >> 3) << 17) |
                            ((uint32_t)(kPBM >> 4) << 24);

// D (TMEM) += A (TMEM, lane = row, 2 bf16 per column) x B (shared, descriptor)
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

// D (TMEM) += A (shared, descriptor) x B (shared, descriptor), both K-major
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

#define SHERRY_TMEM_ST32(taddr, v)                                                                               \
    asm volatile(                                                                                                \
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16," \
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),                        \
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),      \
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),          \
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),         \
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])                      \
        : "memory")

__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

#define SHERRY_TMEM_LD16(taddr, v)                                                                       \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
                 "%15}, [%16];"                                                                          \
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),    \
                   "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), \
                   "=r"(v[14]), "=r"(v[15])                                                               \
                 : "r"(taddr))

#define SHERRY_TMEM_LD32(taddr, v)                                                                               \
    asm volatile(                                                                                                \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17," \
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                                       \
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),        \
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),  \
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),             \
          "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),             \
          "=r"(v[30]), "=r"(v[31])                                                                               \
        : "r"(taddr))

// Arenas (ARN): the same kernel also accumulates X W^T for a dense bf16 latent
// weight W in a third TMEM accumulator and writes Y = (the promoted ternary sum)
// + lambda * that product.  Its W tiles [128 rows x 64 K] come by TMA into the
// same slots as X: a chunk is then two K-steps of X and two of W (64 KB), and the
// ternary A stages shrink to 2 x 2 steps so that the dense accumulator fits in
// TMEM (columns 384..511).
template <int EPI, bool ARN>
__global__ void __launch_bounds__(PRoles<EPI>::kThreads, 1)
k_prefill(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
          const __grid_constant__ PParams P) {
    constexpr int kPTmaWarp = PRoles<EPI>::kTmaWarp, kPMmaWarp = PRoles<EPI>::kMmaWarp;
    constexpr int CS = ARN ? kPArnSteps : kPChunkSteps;   // K-steps per chunk
    constexpr int XS = ARN ? kPArnSlots : kPXSlots;       // chunk slots
    constexpr int AB = ARN ? 2 : kPABuf;                  // A buffers
    constexpr int SLOTB = (ARN ? 2 : 1) * CS * kPStepB;   // bytes per slot (ARN: X, then W tiles)
    constexpr int SPG = CS / kPDecGroups;           // steps each decode group expands per chunk
    constexpr int kWOff = CS * kPStepB;             // W tiles after the X tiles of a slot (ARN)
    constexpr int kDenseCol = kPAcol + AB * CS * kPAcols;  // dense accumulator (ARN)
    static_assert(!ARN || kDenseCol + kPBN <= kPTmemCols, "Arenas plan");
    static_assert(XS * SLOTB <= kPXBytes && XS >= AB + 1 && SLOTB % 1024 == 0, "slot plan");
    extern __shared__ __align__(1024) unsigned char psmem[];
    __shared__ uint64_t bars[2 * kPMaxSlots + kPMaxABuf + 2 * kPAcc + 3];
    __shared__ uint32_t tmem_base_s;
    __shared__ volatile int abort_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t base = (smem_u32(psmem) + 1023u) & ~1023u;
    const uint32_t stX = base;                               // XS slots of SLOTB bytes, 1024-aligned
    const uint32_t table = base + kPXBytes;                  // 256-aligned
    const uint32_t bar0 = smem_u32(&bars[0]);
    auto full_x = [&](int c) { return bar0 + 8u * c; };                    // X (and W) chunk in slot c landed
    auto chunk_empty = [&](int c) { return bar0 + 8u * (XS + c); };  // MMAs of slot c's chunk done
    auto full_a = [&](int h) { return bar0 + 8u * (2 * XS + h); };   // A buffer h written
    auto acc_full = [&](int b) { return bar0 + 8u * (2 * XS + AB + b); };
    auto acc_empty = [&](int b) { return bar0 + 8u * (2 * XS + AB + kPAcc + b); };
    const uint32_t drain = bar0 + 8u * (2 * XS + AB + 2 * kPAcc);  // the MMA thread's last commit
    const uint32_t dense_full = drain + 8u;    // ARN: a tile's dense product is complete
    const uint32_t dense_empty = drain + 16u;  // ARN: the epilogue has read it

    // persistent: tile t = (weight-row tile t % ntn, token tile t / ntn), strided by the grid;
    // chunk and accumulator phases run on across tiles
    const int ntn = (P.N + kPBM - 1) / kPBM;
    const int ntiles = ntn * ((P.M + kPBN - 1) / kPBN);
    const int nk = P.K / kPBK;
    const int nchunks = (nk + CS - 1) / CS;  // the last one may hold fewer steps
    const int gs = P.group_steps;
    const int ngroups = nk / gs;

    if (threadIdx.x == 0) {
        abort_s = 0;
        for (int c = 0; c < XS; ++c) {
            mbar_init(full_x(c), 1);
            mbar_init(chunk_empty(c), 1);
        }
        for (int h = 0; h < AB; ++h) mbar_init(full_a(h), 128 * kPDecGroups);
        for (int b = 0; b < kPAcc; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), 32 * EPI);
        }
        mbar_init(drain, 1);
        mbar_init(dense_full, 1);
        mbar_init(dense_empty, 32 * EPI);
        fence_mbar_init();
    }
    if (threadIdx.x < 32) {
        // bf16 patterns of the 32 block codes (entry = nibble + 16 * sign bit): the
        // low halves (weights 0, 1) and the high halves (weights 2, 3) in separate
        // 128-byte tables, so that a warp's lookups never conflict on a bank
        const uint2 e = decode_block_bf16((uint32_t)threadIdx.x & 15u, (uint32_t)threadIdx.x >> 4);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(table + 4u * threadIdx.x), "r"(e.x) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(table + 128u + 4u * threadIdx.x), "r"(e.y) : "memory");
    }
    if (warp == kPMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                     "r"(kPTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;

    if (warp < EPI) {
        // ---------------- epilogue: row n = tile row 32*(warp%4) + lane, tokens
        // [kCols*(warp/4), kCols*(warp/4) + kCols) of each tile ----------------
        const int q = warp & 3, half = warp >> 2;
        constexpr int kCols = kPBN / (EPI / 4);
        bool ok = true;
        int b = 0;
        uint32_t bph = 0;  // phase parity of accumulator b's use
        uint32_t dph = 0;  // ARN: phase parity of the dense accumulator's use
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const int n = (t % ntn) * kPBM + q * 32 + lane;
            const int m0 = (t / ntn) * kPBN + half * kCols;
            const bool row_ok = n < P.N;
            const bool gsc = !P.row_scale && row_ok;
            const float* srow = P.scales + (int64_t)(row_ok ? n : 0) * P.spr;
            // group scales are loaded two groups ahead of their use
            float a_next = gsc ? __ldg(srow) : 1.0f;
            float a_next2 = (gsc && ngroups > 1) ? __ldg(srow + 1) : 1.0f;
            float acc[kCols];
#pragma unroll
            for (int j = 0; j < kCols; ++j) acc[j] = 0.0f;
            for (int g = 0; g < ngroups; ++g) {
                const float a = a_next;
                a_next = a_next2;
                a_next2 = (gsc && g + 2 < ngroups) ? __ldg(srow + g + 2) : 1.0f;
                ok = mbar_wait(acc_full(b), bph, &abort_s);
                if (!ok) break;
                tc_fence_after();
                const uint32_t t_row = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kPBN + half * kCols);
                // 32 columns per wait (two TMEM loads in flight); the running sums stay in registers
#pragma unroll
                for (int c = 0; c < kCols / 32; ++c) {
                    uint32_t v[16], w[16];
                    SHERRY_TMEM_LD16(t_row + 32 * c, v);
                    SHERRY_TMEM_LD16(t_row + 32 * c + 16, w);
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[32 * c + j] = fmaf(a, __uint_as_float(v[j]), acc[32 * c + j]);
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[32 * c + 16 + j] = fmaf(a, __uint_as_float(w[j]), acc[32 * c + 16 + j]);
                }
                tc_fence_before();
                mbar_arrive(acc_empty(b));
                if (++b == kPAcc) { b = 0; bph ^= 1u; }
            }
            if (!ok) break;
            float a = 1.0f;
            if (P.row_scale && row_ok) a = __ldg(P.scales + (P.per_tensor ? 0 : n));
#pragma unroll
            for (int j = 0; j < kCols; ++j) acc[j] *= a;
            if constexpr (ARN) {
                // Y = the ternary sum + lambda * the dense product
                ok = mbar_wait(dense_full, dph, &abort_s);
                if (!ok) break;
                tc_fence_after();
                const uint32_t t_d = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(kDenseCol + half * kCols);
#pragma unroll
                for (int c = 0; c < kCols / 16; ++c) {
                    uint32_t v[16];
                    SHERRY_TMEM_LD16(t_d + 16 * c, v);
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[16 * c + j] = fmaf(P.lambda, __uint_as_float(v[j]), acc[16 * c + j]);
                }
                tc_fence_before();
                mbar_arrive(dense_empty);
                dph ^= 1u;
            }
            if (row_ok) {
#pragma unroll
                for (int j = 0; j < kCols; ++j) {
                    const int m = m0 + j;
                    if (m < P.M) {
                        const float y = acc[j];
                        if (P.y_bf16)
                            reinterpret_cast<__nv_bfloat16*>(P.Y)[(int64_t)m * P.N + n] = __float2bfloat16_rn(y);
                        else
                            reinterpret_cast<float*>(P.Y)[(int64_t)m * P.N + n] = y;
                    }
                }
            }
        }
    } else if (warp < kPTmaWarp) {
        // ---------------- decode: TMEM lane (= tile row) i per thread; group g expands
        // steps SPG*g .. SPG*g + SPG-1 of every chunk into A buffer (cc % AB) ----------------
        const int g = (warp - EPI) >> 2, q = warp & 3;
        const int i = q * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)kPAcol;
        int cc = 0;  // chunks done so far (all tiles)
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const int n = (t % ntn) * kPBM + i;
            const bool row_ok = n < P.N;
            const uint32_t* idxr = P.idx + (int64_t)(row_ok ? n : 0) * P.words;
            const uint8_t* sgnr = P.sgn + (int64_t)(row_ok ? n : 0) * P.words;
            // ring of the next kPRing chunks' packed words: per step 2 idx words + 2 sign bytes
            uint2 rw[kPRing][2];
            uint32_t rs[kPRing][2];
            auto fetch = [&](int ch, uint2* w, uint32_t* sg) {
#pragma unroll
                for (int e = 0; e < SPG; ++e) {
                    const int ks = ch * CS + SPG * g + e;
                    w[e] = make_uint2(0u, 0u);
                    sg[e] = 0u;
                    if (row_ok && ch < nchunks && ks < nk) {
                        w[e] = __ldg(reinterpret_cast<const uint2*>(idxr + 2 * ks));
                        sg[e] = __ldg(reinterpret_cast<const uint16_t*>(sgnr + 2 * ks));
                    }
                }
            };
#pragma unroll
            for (int r = 0; r < kPRing; ++r) fetch(r, rw[r], rs[r]);
            for (int ch0 = 0; ch0 < nchunks && ok; ch0 += kPRing) {
#pragma unroll
                for (int r = 0; r < kPRing; ++r) {
                    const int ch = ch0 + r;
                    if (ch >= nchunks) break;
                    uint2 w[2] = {rw[r][0], rw[r][1]};
                    uint32_t sb[2] = {rs[r][0], rs[r][1]};
                    fetch(ch + kPRing, rw[r], rs[r]);
                    const int hbuf = cc % AB;
#pragma unroll
                    for (int e = 0; e < SPG; ++e) {
                        const int st = SPG * g + e;
                        if (ch * CS + st >= nk) break;
                        uint32_t v[32];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t wd = h ? w[e].y : w[e].x;
                            const uint32_t sg = (sb[e] >> (8 * h)) & 0xffu;
                            const uint32_t ev = ((wd << 2) & 0x3c3c3c3cu) | (((sg & 0x55u) * 0x01041040u) & 0x40404040u);
                            const uint32_t od = ((wd >> 2) & 0x3c3c3c3cu) | (((sg & 0xaau) * 0x00820820u) & 0x40404040u);
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const uint32_t a = __byte_perm((j & 1) ? od : ev, table, (uint32_t)(j >> 1) | 0x7650u);
                                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v[16 * h + 2 * j]) : "r"(a));
                                asm volatile("ld.shared.u32 %0, [%1+128];" : "=r"(v[16 * h + 2 * j + 1]) : "r"(a));
                            }
                        }
                        // A buffer hbuf was last read by the MMAs of chunk cc - AB, whose
                        // completion the MMA thread commits to that chunk's slot barrier
                        if (e == 0 && cc >= AB) {
                            if (!mbar_wait(chunk_empty((cc - AB) % XS), (uint32_t)(((cc - AB) / XS) & 1),
                                           &abort_s)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        SHERRY_TMEM_ST32(t_lane + (uint32_t)((hbuf * CS + st) * kPAcols), v);
                    }
                    if (!ok) break;
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    mbar_arrive(full_a(hbuf));
                    ++cc;
                }
            }
        }
    } else if (warp == kPTmaWarp) {
        // ---------------- TMA producer for X (and, ARN, the latent-weight tiles) ----------------
        if (lane == 0) {
            int c = 0;
            uint32_t cph = 0;  // phase parity of slot c's use
            int issued[XS] = {};  // chunks loaded into each slot (phases of full_x)
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const int m0 = (t / ntn) * kPBN;
                const int n0 = (t % ntn) * kPBM;
                for (int ch = 0; ch < nchunks; ++ch) {
                    if (!mbar_wait(chunk_empty(c), cph ^ 1u, &abort_s)) {
                        ok = false;
                        break;
                    }
                    const int steps = min(CS, nk - ch * CS);
                    mbar_expect_tx(full_x(c), (uint32_t)(steps * kPStepB * (ARN ? 2 : 1)));
                    for (int st = 0; st < steps; ++st) {
                        tma_load_2d(stX + c * SLOTB + st * kPStepB, &xmap, (ch * CS + st) * kPBK, m0, full_x(c));
                        if constexpr (ARN)
                            tma_load_2d(stX + c * SLOTB + kWOff + st * kPStepB, &wmap, (ch * CS + st) * kPBK, n0,
                                        full_x(c));
                    }
                    ++issued[c];
                    if (++c == XS) { c = 0; cph ^= 1u; }
                }
            }
            // every load issued must land before the CTA's shared memory goes away
            // (after an abort the MMA thread may not have waited for the last ones)
            for (int s = 0; s < XS; ++s)
                if (issued[s] > 0) mbar_drain(full_x(s), (uint32_t)((issued[s] - 1) & 1));
        }
    } else {
        // ---------------- MMA issuer ----------------
        // A single thread issues every MMA, so its own instruction stream is on the
        // critical path: full chunks take an unrolled path, group boundaries are a
        // count-down, and operand addresses are fixed offsets from the chunk base.
        if (lane == 0) {
            int cc = 0, c = 0, b = 0;
            uint32_t cph = 0, bph = 0;
            uint32_t dph = 0;  // ARN: phase parity of the dense accumulator's use
            bool ok = true;
            // one MMA step (K = 64: four K = 16 MMAs) into accumulator b, and (ARN) the
            // dense step into the dense accumulator; returns false on a timed-out wait
            auto step = [&](int& gleft, int ks, uint32_t ta, uint64_t db, uint64_t dw) -> bool {
                const bool first = gleft == gs;
                if (first) {
                    if (!mbar_wait(acc_empty(b), bph ^ 1u, &abort_s)) return false;
                    tc_fence_after();
                }
                const uint32_t td = tmem + (uint32_t)(b * kPBN);
                mma_bf16_ts(td, ta, db, first ? 0u : 1u);
#pragma unroll
                for (int kk = 1; kk < kPBK / 16; ++kk)  // K = 16 per MMA: 8 A columns, +32 bytes in the B row
                    mma_bf16_ts(td, ta + (uint32_t)(8 * kk), db + (uint64_t)(2 * kk), 1u);
                if constexpr (ARN) {
                    if (ks == 0) {
                        if (!mbar_wait(dense_empty, dph ^ 1u, &abort_s)) return false;
                        tc_fence_after();
                    }
                    const uint32_t tdd = tmem + (uint32_t)kDenseCol;
#pragma unroll
                    for (int kk = 0; kk < kPBK / 16; ++kk)
                        mma_bf16_ss(tdd, dw + (uint64_t)(2 * kk), db + (uint64_t)(2 * kk),
                                    (ks == 0 && kk == 0) ? 0u : 1u);
                    if (ks == nk - 1) {
                        mma_commit(dense_full);
                        dph ^= 1u;
                    }
                }
                if (--gleft == 0) {
                    mma_commit(acc_full(b));
                    gleft = gs;
                    if (++b == kPAcc) { b = 0; bph ^= 1u; }
                }
                return true;
            };
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                int gleft = gs;  // steps left in the current group
                for (int ch = 0; ch < nchunks; ++ch, ++cc) {
                    const int hbuf = cc % AB;
                    if (!mbar_wait(full_a(hbuf), (uint32_t)((cc / AB) & 1), &abort_s)) { ok = false; break; }
                    if (!mbar_wait(full_x(c), cph, &abort_s)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t db0 = smem_desc(stX + c * SLOTB);
                    const uint64_t dw0 = smem_desc(stX + c * SLOTB + kWOff);
                    const uint32_t ta0 = tmem + (uint32_t)(kPAcol + hbuf * CS * kPAcols);
                    const int steps = min(CS, nk - ch * CS);
                    if (steps == CS) {
#pragma unroll
                        for (int st = 0; st < CS; ++st)
                            if (!step(gleft, ch * CS + st, ta0 + (uint32_t)(st * kPAcols),
                                      db0 + (uint64_t)((st * kPStepB) >> 4), dw0 + (uint64_t)((st * kPStepB) >> 4))) {
                                ok = false;
                                break;
                            }
                    } else {
                        for (int st = 0; st < steps; ++st)
                            if (!step(gleft, ch * CS + st, ta0 + (uint32_t)(st * kPAcols),
                                      db0 + (uint64_t)((st * kPStepB) >> 4), dw0 + (uint64_t)((st * kPStepB) >> 4))) {
                                ok = false;
                                break;
                            }
                    }
                    if (!ok) break;
                    mma_commit(chunk_empty(c));
                    if (++c == XS) { c = 0; cph ^= 1u; }
                }
            }
            // all MMAs this thread issued complete before TMEM is freed (after an abort
            // no epilogue has waited for them)
            mma_commit(drain);
            mbar_drain(drain, 0u);
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kPMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPTmemCols));
    }
}

// ---- host side -------------------------------------------------------------------

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encode_fn() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

bool prefill_eligible(const ProbShape& s, int64_t M) {
    if (M < 17 || s.N == 0) return false;
    if (s.K % kPBK != 0) return false;
    if (s.granularity == SHERRY_PER_GROUP && s.group % kPBK != 0) return false;
    if (M > (int64_t)0x7fffffff / 2) return false;
    return true;
}

static int encode_2d(CUtensorMap* map, const void* base, int64_t inner, int64_t rows, int box_rows) {
    EncodeTiled enc = encode_fn();
    if (!enc) return SHERRY_ERR_UNSUPPORTED;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kPBK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? SHERRY_OK : SHERRY_ERR_UNSUPPORTED;
}

// Wd: the latent bf16 weight for Arenas (null: the plain linear)
static int prefill_launch_any(const ProbShape& s, const sherry_linear_desc& d, int64_t M, int y_bf16,
                              const uint16_t* Wd, float lambda, cudaStream_t stream) {
    CUtensorMap map, wmap;
    int st = encode_2d(&map, d.X, s.K, M, kPBN);
    if (st) return st;
    if (Wd && (st = encode_2d(&wmap, Wd, s.K, s.N, kPBM))) return st;
    if (!Wd) wmap = map;  // unused
    PParams P{};
    P.idx = d.idx;
    P.sgn = d.sgn;
    P.scales = d.scales;
    P.Y = d.Y;
    P.M = (int)M;
    P.N = (int)s.N;
    P.K = (int)s.K;
    P.words = (int)(s.K / 32);
    P.y_bf16 = y_bf16;
    P.row_scale = s.granularity != SHERRY_PER_GROUP;
    P.per_tensor = s.granularity == SHERRY_PER_TENSOR;
    P.spr = s.granularity == SHERRY_PER_GROUP ? (int)(s.K / s.group) : 1;
    P.group_steps = s.granularity == SHERRY_PER_GROUP ? s.group / kPBK : (int)(s.K / kPBK);
    P.lambda = lambda;
    // per device: the shared-memory opt-in of every instantiation, and the SM count
    static PerDevice dev_sms;
    int sms = 0;
    st = per_device(dev_sms, &sms, [](int& v) {
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_prefill<8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem));
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_prefill<16, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem));
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_prefill<8, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem));
        SHERRY_CUDA_CHECK(cudaFuncSetAttribute(k_prefill<16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem));
        int dev = 0;
        SHERRY_CUDA_CHECK(cudaGetDevice(&dev));
        SHERRY_CUDA_CHECK(cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev));
        if (v < 1) v = 1;
        return SHERRY_OK;
    });
    if (st) return st;
    const int64_t tiles = ((s.N + kPBM - 1) / kPBM) * ((M + kPBN - 1) / kPBN);
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    // 16 epilogue warps (32 token columns each) drain a group accumulator faster; measured on the
    // 3B shapes that pays for group scales up to K = 4096 (+6%) and costs at K = 8192 (-15%) and
    // for per-row scales (one drain per tile; -1.5% at 2048 and 4096 tokens)
    const bool epi16 = s.granularity == SHERRY_PER_GROUP && s.K <= 4096;
    if (Wd) {
        if (epi16)
            k_prefill<16, true><<<grid, PRoles<16>::kThreads, kPSmem, stream>>>(map, wmap, P);
        else
            k_prefill<8, true><<<grid, PRoles<8>::kThreads, kPSmem, stream>>>(map, wmap, P);
    } else {
        if (epi16)
            k_prefill<16, false><<<grid, PRoles<16>::kThreads, kPSmem, stream>>>(map, wmap, P);
        else
            k_prefill<8, false><<<grid, PRoles<8>::kThreads, kPSmem, stream>>>(map, wmap, P);
    }
    SHERRY_LAUNCH_CHECK();
    return SHERRY_OK;
}

int prefill_launch(const ProbShape& s, const sherry_linear_desc& d, int64_t M, int y_bf16, cudaStream_t stream) {
    return prefill_launch_any(s, d, M, y_bf16, nullptr, 0.0f, stream);
}

bool arenas_eligible(const ProbShape& s, int64_t M) {
    if (M < 1 || s.N == 0 || s.K % kPBK != 0) return false;
    if (s.granularity == SHERRY_PER_GROUP && s.group % kPBK != 0) return false;
    return M <= (int64_t)0x7fffffff / 2 && s.N <= (int64_t)0x7fffffff / 2;
}

int arenas_launch(const ProbShape& s, const sherry_linear_desc& d, int64_t M, int y_bf16, const uint16_t* Wd,
                  float lambda, cudaStream_t stream) {
    return prefill_launch_any(s, d, M, y_bf16, Wd, lambda, stream);
}

int device_status_take(cudaStream_t stream) {
    SHERRY_CUDA_CHECK(cudaStreamSynchronize(stream));
    int v = 0;
    SHERRY_CUDA_CHECK(cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)));
    if (v) {
        const int zero = 0;
        SHERRY_CUDA_CHECK(cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)));
    }
    const int w = skinny_status_take();
    const int x = stream_status_take();
    return v ? v : w ? w : x;
}

}  // namespace sherry
