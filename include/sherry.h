/*
 * sherry.h -- C ABI of the B200 (sm_100a) library for Sherry 3:4-sparse
 * ternary (1.25-bit) weights: quantise+pack, packed linear, unpack.
 *
 * The method (page "Sherry: Hardware-Efficient 1.25-Bit Ternary Quantization
 * via Fine-grained Sparsification", digest paragraphs on the 3:4 rule, on
 * greedy Sparse-AbsMean and on inference; page "Sherry, Tequila and Fairies in
 * Python", section 1.1 Sherry Quantization):
 *   - in every block of 4 consecutive weights along K exactly one weight is 0
 *     (the smallest |w|) and the other three are +-1 (their signs);
 *   - the scale alpha of a domain (a group of `group` weights along K, a row,
 *     or the whole tensor) is the mean |w| of the kept weights;
 *   - each block is stored in 5 bits, 1 sign bit + 4 lookup bits (32 states);
 *   - the layer computes Y = X (T alpha)^T.
 *
 * Readings fixed by this library where the pages are silent:
 *   - the lowest index is zeroed when several |w| tie for the minimum;
 *   - sign(w) = +1 for w >= 0, -0.0 included;
 *   - nibble = 4*z + 2*d1 + d2 (z = zero position; p0 < p1 < p2 the kept
 *     positions; d1 = [s(p1) != s(p0)], d2 = [s(p2) != s(p0)]); sign bit
 *     G = [s(p0) < 0];
 *   - alpha = S / D in fp32 with S the adjacent-pairwise fp32 sum of the kept
 *     |w| over the domain in K order (the domain padded with +0.0 to a power of
 *     two; the zeroed weight contributes +0.0), D = fp32(L*3/4) for a domain of
 *     L weights (D = 1 for an empty tensor), one IEEE division, no flush to zero;
 *   - no bias term.
 *
 * PACKED LAYOUT (device memory, row-major planes, little-endian):
 *   idx    uint32 [N][K/32]  nibble of block j (weights 4j..4j+3 of the word's
 *                            32) at bits 4j..4j+3
 *   sgn    uint8  [N][K/32]  bit j = G of block j
 *   scales float  [num]      per-group [N][K/group], per-channel [N], per-tensor [1]
 *   => 1.25 bit/weight for idx+sgn, plus 32 bits per scale domain.
 *
 * CONVENTIONS
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise; the
 *     caller allocates (and owns) every buffer.  `stream` is a cudaStream_t
 *     (NULL = legacy default stream).  Calls are asynchronous on `stream`.
 *   - Arguments are validated on the host before any launch; on an error
 *     nothing is launched and nothing is written.
 *   - Inputs must be finite; non-finite weights or activations give
 *     unspecified (but memory-safe) results.
 *   - Shapes: N >= 0, M >= 0 (0 = nothing to do), 32 <= K <= SHERRY_MAX_K,
 *     K % 32 == 0; per-group needs group > 0, group % 32 == 0, K % group == 0.
 *   - Alignment: W, X, Y, W_out, idx, sgn and scales 16-byte aligned (else
 *     SHERRY_ERR_ALIGN): the kernels copy them in 16-byte pieces.
 *   - Results are deterministic: the same call on the same inputs gives the
 *     same bits (no float atomics; every reduction has a fixed order).
 */
#ifndef SHERRY_H
#define SHERRY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define SHERRY_OK 0
#define SHERRY_ERR_NULL 1          /* a required pointer is NULL */
#define SHERRY_ERR_SHAPE 2         /* bad N, K or M */
#define SHERRY_ERR_GRANULARITY 3   /* unknown granularity */
#define SHERRY_ERR_GROUP 4         /* bad group size for per-group */
#define SHERRY_ERR_DTYPE 5         /* unknown element type */
#define SHERRY_ERR_ALIGN 6         /* misaligned pointer */
#define SHERRY_ERR_WORKSPACE 7     /* workspace missing or too small */
#define SHERRY_ERR_CUDA 8          /* a CUDA call or launch failed (see sherry_last_cuda_error) */
#define SHERRY_ERR_TIMEOUT 9       /* a bounded device wait gave up */
#define SHERRY_ERR_UNSUPPORTED 10  /* valid request the library cannot run here (e.g. no sm_100 device) */

/* granularity of alpha */
#define SHERRY_PER_TENSOR 0
#define SHERRY_PER_CHANNEL 1
#define SHERRY_PER_GROUP 2

/* element types */
#define SHERRY_F32 0
#define SHERRY_BF16 1

/* operations, for sherry_workspace_bytes */
#define SHERRY_OP_QUANTIZE_PACK 0
#define SHERRY_OP_LINEAR 1
#define SHERRY_OP_UNPACK 2

#define SHERRY_MAX_K 262144

/* ---- sizes ------------------------------------------------------------- */

/* bytes of the idx plane, N*K/8 (0 on invalid shape) */
size_t sherry_idx_bytes(int64_t N, int64_t K);
/* bytes of the sgn plane, N*K/32 (0 on invalid shape) */
size_t sherry_sgn_bytes(int64_t N, int64_t K);
/* number of fp32 scales: N*K/group, N or 1 (-1 on invalid arguments) */
int64_t sherry_num_scales(int64_t N, int64_t K, int granularity, int group);
/* device workspace an operation needs (0 = none); pass at least this many
 * bytes.  A linear workspace starts with a 256 KiB region of split-K tickets
 * that must be zero before its first use; every call that returns SHERRY_OK
 * leaves that region zero (what follows it is scratch).  One workspace may be
 * shared by linear calls (single or batched) that do not overlap on the device;
 * do not share it with the quantise+pack scratch. */
size_t sherry_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int granularity, int group);

/* ---- quantise + pack ----------------------------------------------------
 * Greedy Sparse-AbsMean ("Sherry: ... Fine-grained Sparsification", digest
 * paragraph on the 3:4 rule and quantisation; "Sherry, Tequila and Fairies in
 * Python" section 1.1, the N:M quantiser with n=3, m=4 and its granularities).
 *   W        [N][K] row-major, fp32 or bf16 (w_dtype); read only
 *   idx,sgn  packed planes (layout above); fully overwritten
 *   scales   sherry_num_scales(...) floats; fully overwritten
 *   workspace  sherry_workspace_bytes(SHERRY_OP_QUANTIZE_PACK, 0, N, K, g, group)
 *            bytes (per-tensor only; NULL/0 otherwise)
 * Output is bit-identical to the definition above. */
int sherry_quantize_pack(const void* W, int w_dtype, int64_t N, int64_t K, int granularity, int group,
                         uint32_t* idx, uint8_t* sgn, float* scales,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ---- fake quantisation (the quantiser's forward output, for QAT) -----------
 * "Sherry, Tequila and Fairies in Python", section 1.1 (SherryNMQuant.forward
 * and SherryLinear): W_q = sign(w) * mask * alpha, i.e. t[n][k] * alpha(n,k),
 * written together with the packed planes and scales of sherry_quantize_pack
 * (same arguments, same workspace, bit-identical planes and scales).
 *   Wq       [N][K] fp32 (wq_dtype SHERRY_F32: t * alpha exactly) or bf16
 *            (SHERRY_BF16: round to nearest even of t * alpha); fully overwritten
 * Group and row scales: one pass over W (the row's Wq is written from its packed
 * words once its scales are known).  Per-tensor: the scale needs the whole
 * tensor, so Wq is written by a second pass over the packed planes.
 * The straight-through estimator's backward is the identity (the gradient with
 * respect to W_q is the gradient with respect to W): it needs no kernel. */
int sherry_fake_quant(const void* W, int w_dtype, int64_t N, int64_t K, int granularity, int group,
                      void* Wq, int wq_dtype, uint32_t* idx, uint8_t* sgn, float* scales,
                      void* workspace, size_t workspace_bytes, void* stream);

/* ---- Tequila-style dead-weight term ----------------------------------------
 * "Sherry, Tequila and Fairies in Python", sections 1.2 and 2.1 (UltraQuantV2,
 * UltraQuantLinear): the weights a ternary quantiser zeroes are kept as
 * B = eps * w and add F.linear(ones, B) or F.linear(sign(x), B) to the layer.
 * Here the zeroed weights are Sherry's (the smallest |w| of every block of 4).
 * sherry_quantize_pack_tequila quantises and packs as sherry_quantize_pack (same
 * planes, scales, workspace) and, in the same pass over W, writes
 *   D      bf16 [N][K/4]: round-to-nearest-even of the fp32 product eps * w at
 *          the zeroed position of each block (16-byte aligned)
 *   bias   fp32 [N] (optional, NULL: none): the canonical pairwise fp32 sum of
 *          the row's D values = F.linear(ones, B)
 * sherry_linear_tequila computes Y = X (T alpha)^T + term with
 *   mode SHERRY_TEQUILA_ONES: term[m][n] = bias[n]
 *   mode SHERRY_TEQUILA_SIGN: term[m][n] = sum_b sign(X[m][4b + z(n,b)]) D[n][b]
 *        (sign(0) = 0), z the zero position recorded in idx
 * the linear by its usual kernel into fp32, then one term pass (fp32; Y fp32 or
 * bf16, round to nearest even of the sum).
 *   workspace  sherry_linear_tequila_workspace_bytes(M, N, K, g, group, y_dtype) bytes
 *            (the linear's ticket contract: the first 256 KiB zero on entry and left
 *            zero; bf16 Y adds M*N fp32 scratch after max(the linear's bytes, 256 KiB)) */
#define SHERRY_TEQUILA_ONES 0
#define SHERRY_TEQUILA_SIGN 1
int sherry_quantize_pack_tequila(const void* W, int w_dtype, int64_t N, int64_t K, int granularity, int group,
                                 float eps, uint32_t* idx, uint8_t* sgn, float* scales, uint16_t* D, float* bias,
                                 void* workspace, size_t workspace_bytes, void* stream);
int sherry_linear_tequila(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                          const uint32_t* idx, const uint8_t* sgn, const float* scales, int granularity, int group,
                          const uint16_t* D, const float* bias, int mode,
                          void* Y, int y_dtype, void* workspace, size_t workspace_bytes, void* stream);
size_t sherry_linear_tequila_workspace_bytes(int64_t M, int64_t N, int64_t K, int granularity, int group,
                                             int y_dtype);

/* One weight of a batched quantise + pack (all pointers device pointers). */
typedef struct sherry_quantize_desc {
    const void* W;          /* [N][K], w_dtype */
    uint32_t* idx;
    uint8_t* sgn;
    float* scales;
    void* Wq;               /* optional fake-quantised output [N][K] in wq_dtype (NULL: none) */
    int64_t N, K;
    int32_t w_dtype, granularity, group, wq_dtype;
} sherry_quantize_desc;

/* ---- batched quantise + pack ----------------------------------------------
 * `count` independent weights (count <= SHERRY_MAX_BATCH; any mix of element
 * types and granularities) in one launch of the quantise kernel, plus one launch
 * that finalises every per-tensor scale (and, for per-tensor weights with Wq, one
 * pass that writes Wq).  Each desc's outputs are bit-identical to the single
 * call's.  `descs` is a HOST array read during the call only.
 *   workspace  sherry_quantize_pack_batched_workspace_bytes(descs, count) bytes
 *            (per-tensor weights only; 256-byte aligned) */
int sherry_quantize_pack_batched(const sherry_quantize_desc* descs, int count,
                                 void* workspace, size_t workspace_bytes, void* stream);
size_t sherry_quantize_pack_batched_workspace_bytes(const sherry_quantize_desc* descs, int count);

/* ---- packed linear -------------------------------------------------------
 * Y[m][n] = sum_k X[m][k] * t[n][k] * alpha(n,k)  ("Sherry: ..." digest: Y = X T alpha;
 * inference builds lookup tables from the activations, accumulates, then applies
 * the scale; "Sherry, Tequila and Fairies in Python" section 1.1: F.linear(x, w)).
 *   X        bf16 [M][K] row-major (uint16 storage); read only
 *   idx,sgn,scales  packed weight of shape [N][K] with (granularity, group)
 *   Y        [M][N] row-major, fp32 or bf16 (y_dtype, round to nearest even);
 *            fully overwritten
 *   workspace  sherry_workspace_bytes(SHERRY_OP_LINEAR, M, N, K, g, group) bytes
 * fp32 accumulation; alpha applied once per group (or row).  Kernels:
 * M <= 16 with K % 512 == 0 (group 128 or 256, per-channel or per-tensor) a
 * warp-specialised streaming kernel (lookup tables for M <= 2, tensor-core
 * consumers from M = 3); other 2 <= M <= 8 with
 * K % 128 == 0 a warp-level tensor-core (mma.sync) kernel; 9 <= M <= 32 with K % 256 == 0 and
 * (per-group) group % 64 == 0 a tensor-core (tcgen05) kernel for few tokens;
 * M >= 17 with K % 64 == 0 and group % 64 == 0 the tcgen05 prefill kernel;
 * anything else the general lookup-table kernel (any M). */
int sherry_linear(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                  const uint32_t* idx, const uint8_t* sgn, const float* scales,
                  int granularity, int group,
                  void* Y, int y_dtype, void* workspace, size_t workspace_bytes, void* stream);

/* One independent linear of a batch (all pointers device pointers). */
typedef struct sherry_linear_desc {
    const uint16_t* X;      /* bf16 [M][K] */
    const uint32_t* idx;
    const uint8_t* sgn;
    const float* scales;
    void* Y;                /* [M][N], y_dtype of the batch call */
    int64_t N, K;
    int32_t granularity, group;
} sherry_linear_desc;

#define SHERRY_MAX_BATCH 256

/* ---- batched packed linear ----------------------------------------------
 * `count` independent linears with the same M in one call, e.g. the
 * projections of a decoder layer stack for one token.  Each desc is computed
 * as by sherry_linear, by the kernel that sherry_linear would pick for it
 * (except that the streaming kernel's problems go to the others when the whole
 * batch has more row blocks than its tickets): the problems that share a kernel
 * share one launch of it (each prefill problem, M >= 17, gets a launch of its
 * own; several such launches run on four library-owned side streams per device,
 * forked from `stream` and joined back into it with events, so `stream`'s order
 * and graph capture hold).  Y agrees with sherry_linear's within the fp32
 * summation-order bound; the streaming kernels (1 to 16 tokens) split K where the
 * batch as a whole balances best, so they are not bit-identical to a single call.  A call
 * repeated with the same arguments gives bit-identical Y.  `descs` is a HOST
 * array, read during the call only.  count <= SHERRY_MAX_BATCH.
 *   workspace  sherry_linear_batched_workspace_bytes(descs, count, M) bytes. */
int sherry_linear_batched(const sherry_linear_desc* descs, int count, int64_t M, int y_dtype,
                          void* workspace, size_t workspace_bytes, void* stream);
size_t sherry_linear_batched_workspace_bytes(const sherry_linear_desc* descs, int count, int64_t M);

/* ---- Arenas training linear ------------------------------------------------
 * "Sherry: ... Fine-grained Sparsification", digest paragraph on Arenas: during
 * quantisation-aware training the layer adds an annealed full-precision
 * residual, Y = X T alpha + lambda_t X W, with lambda_t decayed to 0 by a cosine;
 * at inference it is gone.  One kernel computes both products on the tensor
 * cores (the ternary one with alpha promoted per group in fp32, the dense one in
 * its own fp32 accumulator) and writes Y = ternary + lambda * dense.
 *   Wd       the latent weight, bf16 [N][K] row-major (16-byte aligned)
 *   other arguments as sherry_linear (no workspace); needs K % 64 == 0 and, for
 *   group scales, group % 64 == 0 (else SHERRY_ERR_UNSUPPORTED).
 * sherry_arenas_lambda: lambda0 * (1 + cos(pi * min(step, total) / total)) / 2. */
int sherry_arenas_linear(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                         const uint32_t* idx, const uint8_t* sgn, const float* scales, int granularity, int group,
                         const uint16_t* Wd, float lambda, void* Y, int y_dtype, void* stream);
float sherry_arenas_lambda(int64_t step, int64_t total, float lambda0);

/* ---- chained linears (dependent phases) -----------------------------------
 * `count` linears with the same M (e.g. one decode token through a layer
 * stack) grouped into n_phases phases: phase p holds descs[phase_begin[p] ..
 * phase_begin[p+1]) (phase_begin: HOST array of n_phases + 1 indices,
 * phase_begin[0] = 0, non-decreasing, phase_begin[n_phases] = count).  The
 * linears of a phase are independent; every linear of phase p+1 starts after
 * every linear of phase p has written Y, so a later phase may read an earlier
 * phase's Y as its X (bf16 Y, y_dtype SHERRY_BF16, read in place).  Each Y is
 * computed as by sherry_linear (fp32 accumulation, alpha once per group), within
 * the fp32 summation-order bound of it.
 *   One to three tokens with every K % 512 == 0, or four tokens with every
 *   K % 256 == 0, and group 128 or 256 (or row scales): one cooperative launch
 *   (one CTA per SM, all resident) in which a grid-wide bounded barrier
 *   separates the phases and the packed weights of the next phase stream in
 *   while it resolves ("Sherry: ..." digest: inference streams the packed
 *   weights through lookup tables; the pages' layer is F.linear).  One and two
 *   tokens give each CTA whole 32-row blocks over all of K (the K sum stays in
 *   the CTA, in a fixed order); three and four tokens split row blocks over CTAs
 *   as the batched launch does.  Otherwise: one sherry_linear_batched-style
 *   launch set per phase, ordered by the stream.
 *   workspace  sherry_linear_chain_workspace_bytes(...) bytes; the same ticket
 *            contract as a linear workspace (first 256 KiB zero before the first
 *            use; every successful call leaves it zero). */
int sherry_linear_chain(const sherry_linear_desc* descs, int count, const int* phase_begin, int n_phases,
                        int64_t M, int y_dtype, void* workspace, size_t workspace_bytes, void* stream);
size_t sherry_linear_chain_workspace_bytes(const sherry_linear_desc* descs, int count, const int* phase_begin,
                                           int n_phases, int64_t M);

/* ---- packed linear without a workspace -------------------------------------
 * No counterpart on the pages: this is a service for callers that cannot
 * allocate device memory (a host framework that plans all memory ahead and
 * hands a kernel only its inputs and outputs, a plugin interface without a
 * scratch argument, a latency-critical path that must not enter the
 * allocator).  Same arguments and result as sherry_linear, minus the
 * workspace.  Its scratch is a fixed device array of
 * SHERRY_NOALLOC_SCRATCH_BYTES inside the library, held by every GPU that loads
 * the library until the process exits; a call that would need more returns
 * SHERRY_ERR_WORKSPACE.  The first call on a device looks up the array's device
 * address (make that first call before any stream capture).  Every call zeroes
 * the array's ticket region on `stream` before its kernel and otherwise reuses
 * what the previous call left; all calls share the one array, so calls that
 * overlap on the GPU (other streams, other host threads) race -- keep them
 * ordered.  Nothing is allocated or freed. */
#define SHERRY_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)  /* one problem's largest plan on up to 224 SMs
                                                           (checked at compile time for each plan) */
int sherry_linear_noalloc(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                          const uint32_t* idx, const uint8_t* sgn, const float* scales,
                          int granularity, int group, void* Y, int y_dtype, void* stream);

/* ---- unpack ----------------------------------------------------------------
 * Dense bf16 W_out[n][k] = round_to_nearest_even(t[n][k] * alpha(n,k)); the
 * inverse of the 5-bit code (32 states, "Sherry: ..." digest) times the scale.
 *   W_out    bf16 [N][K] (uint16 storage); fully overwritten */
int sherry_unpack(const uint32_t* idx, const uint8_t* sgn, const float* scales,
                  int64_t N, int64_t K, int granularity, int group,
                  uint16_t* W_out, void* stream);

/* One weight of a batched unpack (all pointers device pointers). */
typedef struct sherry_unpack_desc {
    const uint32_t* idx;
    const uint8_t* sgn;
    const float* scales;
    int64_t N, K;
    int32_t granularity, group;
    uint16_t* W_out;        /* bf16 [N][K] */
} sherry_unpack_desc;

/* ---- batched unpack ---------------------------------------------------------
 * `count` independent unpacks (count <= SHERRY_MAX_BATCH) in one launch, each
 * exactly as by sherry_unpack (bit-identical W_out).  `descs` is a HOST array,
 * read during the call only.  Each desc is validated like the arguments of
 * sherry_unpack; on an error nothing is launched. */
int sherry_unpack_batched(const sherry_unpack_desc* descs, int count, void* stream);

/* ---- diagnostics ----------------------------------------------------------- */
const char* sherry_status_string(int status);
/* cudaError_t value behind the last SHERRY_ERR_CUDA returned on this thread */
int sherry_last_cuda_error(void);
/* Synchronises `stream`, then returns SHERRY_ERR_TIMEOUT if a bounded device
 * wait of a tensor-core kernel or of the streaming decode kernel gave up since
 * the previous query (its outputs are then invalid), else SHERRY_OK; clears the
 * flag.  SHERRY_ERR_CUDA if the synchronisation fails.  After SHERRY_ERR_TIMEOUT
 * the split-K tickets of the linear workspace used by the failed call may be
 * left nonzero: zero its first 256 KiB (or take a fresh zeroed workspace)
 * before the next linear call with it. */
int sherry_device_status(void* stream);
/* How many nonzero statuses sherry_device_status has returned in this process
 * (a host-side count, no device work).  A caller that caches workspaces
 * compares it with the value it saw when it last zeroed them: a change means a
 * wait gave up since, and the cached ticket regions must be zeroed again. */
int64_t sherry_timeout_count(void);
/* Budget, in SM clock cycles, of every bounded wait of the streaming decode
 * kernels (1 to 16 tokens, and chained launches), for launches made after this call; cycles <= 0
 * restores the default (4e9, about 2 s at the boost clock).  Returns the previous
 * budget.  Meant for exercising the failure path: with a budget of a few cycles
 * the waits give up, the call's outputs are invalid, and sherry_device_status
 * reports SHERRY_ERR_TIMEOUT.  These kernels hold no tensor memory (their
 * tensor-core form multiplies with mma.sync in registers) and issue only
 * cp.async copies, which they complete before exiting, so the context stays
 * usable.  The tcgen05 kernels keep the default budget. */
int64_t sherry_set_wait_budget(int64_t cycles);
/* library version, e.g. 0x000100 = 0.1.0 */
int sherry_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SHERRY_H */
