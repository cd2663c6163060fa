// common.cuh -- internal helpers shared by the library's CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "sherry.h"

namespace sherry {

constexpr unsigned kFull = 0xffffffffu;

// last CUDA error seen by an entry point on this host thread
void set_cuda_error(cudaError_t e);

#define SHERRY_CUDA_CHECK(expr)                              \
    do {                                                     \
        cudaError_t _e = (expr);                             \
        if (_e != cudaSuccess) {                             \
            ::sherry::set_cuda_error(_e);                    \
            return SHERRY_ERR_CUDA;                          \
        }                                                    \
    } while (0)

#define SHERRY_LAUNCH_CHECK() SHERRY_CUDA_CHECK(cudaGetLastError())

// One value per device, computed on first use with that device current.  Kernel
// attributes (the opt-in to more than 48 KB of dynamic shared memory), occupancies
// and device properties belong to a device: a process-wide flag would skip them
// on the second GPU a process uses.
struct PerDevice {
    std::mutex mu;
    std::vector<int> val;  // 0 = not computed yet
};

// *out = pd's value for the current device; `init(int& v)` computes it the first
// time (returns a status; v must be nonzero on success).
template <class F>
inline int per_device(PerDevice& pd, int* out, F&& init) {
    int dev = 0;
    SHERRY_CUDA_CHECK(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lk(pd.mu);
    if ((int)pd.val.size() <= dev) pd.val.resize(dev + 1, 0);
    if (pd.val[dev] == 0) {
        int v = 0;
        const int st = init(v);
        if (st) return st;
        pd.val[dev] = v;
    }
    *out = pd.val[dev];
    return SHERRY_OK;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__host__ __device__ __forceinline__ int64_t pow2_ceil64(int64_t x) {
    int64_t p = 1;
    while (p < x) p <<= 1;
    return p;
}

__host__ __device__ __forceinline__ int ilog2_exact(int64_t x) {  // -1 if not a power of two
    if (x <= 0 || (x & (x - 1))) return -1;
    int s = 0;
    while ((int64_t(1) << s) < x) ++s;
    return s;
}

// Canonical pairwise sum of v[0..n) (adjacent pairs, padded with +0.0 to a
// power of two), evaluated sequentially with a stack of completed subtrees.
// Every value here is >= 0, so adding a padding zero is exact and the padded
// tree equals the right fold of the stack.
__device__ __forceinline__ float tree_sum_seq(const float* v, int n) {
    float st[32];
    int lv[32];
    int top = 0;
    for (int i = 0; i < n; ++i) {
        float x = v[i];
        int l = 0;
        while (top > 0 && lv[top - 1] == l) {
            x = st[top - 1] + x;
            --top;
            ++l;
        }
        st[top] = x;
        lv[top] = l;
        ++top;
    }
    if (top == 0) return 0.0f;
    float r = st[top - 1];
    for (int t = top - 2; t >= 0; --t) r = st[t] + r;
    return r;
}

// The same canonical sum for n <= 8 (n <= 16), in registers: padding to 8 (16)
// adds whole zero subtrees, which is exact for values >= 0, so the result equals
// the tree over the next power of two of n.
__device__ __forceinline__ float tree_sum8(const float* v, int n) {
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = i < n ? v[i] : 0.0f;
    return ((x[0] + x[1]) + (x[2] + x[3])) + ((x[4] + x[5]) + (x[6] + x[7]));
}
__device__ __forceinline__ float tree_sum16(const float* v, int n) {
    const float a = tree_sum8(v, n < 8 ? n : 8);
    const float b = n > 8 ? tree_sum8(v + 8, n - 8) : 0.0f;
    return a + b;
}

// Canonical pairwise sum of v[0..n) by one full warp; the result is returned in
// every lane.  Each lane reduces an aligned power-of-two segment sequentially,
// then the xor butterfly (offsets 1, 2, 4, ...) combines adjacent segments,
// which is exactly the upper levels of the same tree.
__device__ __forceinline__ float warp_tree_sum(const float* v, int n) {
    const int lane = threadIdx.x & 31;
    int64_t P = pow2_ceil64(n > 0 ? n : 1);
    float x;
    int span;  // number of lanes that carry tree nodes
    if (P <= 32) {
        x = (lane < n) ? v[lane] : 0.0f;
        span = (int)P;
    } else {
        int seg = (int)(P / 32);
        int lo = lane * seg;
        int cnt = n - lo;
        cnt = cnt < 0 ? 0 : (cnt > seg ? seg : cnt);
        x = seg <= 8 ? tree_sum8(v + lo, cnt) : seg <= 16 ? tree_sum16(v + lo, cnt) : tree_sum_seq(v + lo, cnt);
        span = 32;
    }
    for (int off = 1; off < span; off <<= 1) x = x + __shfl_xor_sync(kFull, x, off);
    return __shfl_sync(kFull, x, 0);
}

// Linear workspaces start with a fixed region of split-K tickets, shared by
// every decode kernel: tickets must be zero before a call and each call leaves
// them zero; partial sums always live after this region, so calls that take
// different kernels can share one workspace.
constexpr size_t kTicketBytes = 256 * 1024;
constexpr int kMaxTickets = (int)(kTicketBytes / sizeof(int));

struct ProbShape {
    int64_t N, K;
    int granularity, group;
};

// One weight to quantise and pack (quantize.cu); Wq, if not null, also receives
// the fake-quantised weights t * alpha in wq_dtype.
struct QuantizeJob {
    const void* W;
    int w_dtype;
    int64_t N, K;
    int granularity, group;
    uint32_t* idx;
    uint8_t* sgn;
    float* scales;
    void* Wq;
    int wq_dtype;
    uint16_t* D;   // optional Tequila-style dead-weight plane, bf16 [N][K/4]
    float* bias;   // optional row sums of D, fp32 [N]
    float eps;
};

// launchers (quantize.cu, unpack.cu, gemv.cu)
size_t quantize_workspace_bytes(int64_t N, int64_t K, int granularity);
size_t quantize_batch_workspace_bytes(const QuantizeJob* jobs, int count);
int quantize_jobs_launch(const QuantizeJob* jobs, int count, void* workspace, int sms, cudaStream_t stream);
int unpack_launch(const sherry_unpack_desc* descs, int count, cudaStream_t stream, int num_sms);
// f32[i] != 0: problem i's W_out is fp32 t * alpha instead of bf16
int unpack_launch_ex(const sherry_unpack_desc* descs, const int* f32, int count, cudaStream_t stream, int num_sms);
size_t lut_workspace_bytes(const ProbShape* shapes, int count, int64_t M, int sms);
int lut_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M,
                      int y_bf16, void* workspace, int sms, cudaStream_t stream);
// tensor-core prefill kernel (prefill.cu)
bool prefill_eligible(const ProbShape& s, int64_t M);
int prefill_launch(const ProbShape& s, const sherry_linear_desc& d, int64_t M, int y_bf16, cudaStream_t stream);
int device_status_take(cudaStream_t stream);
// Arenas training linear on the prefill kernel: Y = X (T alpha)^T + lambda X Wd^T (prefill.cu)
bool arenas_eligible(const ProbShape& s, int64_t M);
int arenas_launch(const ProbShape& s, const sherry_linear_desc& d, int64_t M, int y_bf16, const uint16_t* Wd,
                  float lambda, cudaStream_t stream);
// few-token tensor-core kernel (gemv_tc.cu)
bool hmma_eligible(const ProbShape& s, int64_t M);
int hmma_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                       cudaStream_t stream);
bool skinny_eligible(const ProbShape& s, int64_t M);
int skinny_status_take();  // SHERRY_ERR_TIMEOUT if a bounded wait gave up since the last call
int skinny_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                         int sms, cudaStream_t stream);
// one- and two-token streaming kernel (gemv_stream.cu)
bool stream_eligible(const ProbShape& s, int64_t M);
bool mstream_eligible(const ProbShape& s, int64_t M);  // 3..16 tokens, tensor-core consumers
int mstream_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                          void* workspace, int sms, cudaStream_t stream);
int64_t stream_tiles(const ProbShape& s);  // row blocks (tickets) of one problem
int stream_status_take();                   // SHERRY_ERR_TIMEOUT if a bounded wait gave up since the last call
long long stream_set_wait_cycles(long long cycles);  // returns the previous budget; <= 0 restores the default
size_t stream_workspace_bytes(const ProbShape* shapes, int count, int64_t M, int sms);
int stream_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                         void* workspace, int sms, cudaStream_t stream);
// Tequila-style dead-weight term added to an fp32 linear output (tequila.cu):
// mode 0 Y = Yin + bias[n], mode 1 Y = Yin + sign(X) D^T
int tequila_term_launch(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* idx, const uint16_t* D,
                        const float* bias, int mode, const float* Yin, void* Y, int y_bf16, cudaStream_t stream);
// chained phases on the streaming kernel (cooperative launch, one CTA per SM)
bool chain_eligible(const ProbShape& s, int64_t M);
bool chain_launch_ok(const ProbShape* shapes, int count, int n_phases, int64_t M);
size_t chain_workspace_bytes(const ProbShape* shapes, int count, const int* phase_begin, int n_phases, int64_t M,
                             int sms);
int chain_linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, const int* phase_begin,
                        int n_phases, int64_t M, int y_bf16, void* workspace, int sms, cudaStream_t stream);

}  // namespace sherry
