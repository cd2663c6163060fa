// api.cu -- the library's C ABI (declared in include/sherry.h): argument checks
// on the host, then the launches.  Nothing here allocates device memory.
#include "common.cuh"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <vector>

namespace sherry {

static thread_local int g_last_cuda_error = 0;
void set_cuda_error(cudaError_t e) { g_last_cuda_error = (int)e; }

// number of SMs of the current device (cached per device)
static int device_sms() {
    static std::mutex mu;
    static std::vector<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    std::lock_guard<std::mutex> lk(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
    if (cache[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cache[dev] = v;
    }
    return cache[dev];
}

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Side streams for the prefill launches of one batched call, per device.  The
// problems are independent linears, each a persistent grid over its own tiles; a
// small one leaves SMs idle that the next one's CTAs can take if the launches
// run on different streams.  They are forked from the caller's stream and joined
// back into it with events, so stream order and graph capture hold.
constexpr int kForkStreams = 4;
struct ForkPool {
    cudaStream_t s[kForkStreams];
    cudaEvent_t fork, join[kForkStreams];
    bool ready = false;
};
static std::mutex g_fork_mu;  // held for a whole fork/join (host-side enqueue only)
static std::vector<ForkPool> g_fork;

static int fork_pool(ForkPool** out) {
    int dev = 0;
    SHERRY_CUDA_CHECK(cudaGetDevice(&dev));
    if ((int)g_fork.size() <= dev) g_fork.resize(dev + 1);
    ForkPool& fp = g_fork[dev];
    if (!fp.ready) {
        for (int k = 0; k < kForkStreams; ++k) {
            SHERRY_CUDA_CHECK(cudaStreamCreateWithFlags(&fp.s[k], cudaStreamNonBlocking));
            SHERRY_CUDA_CHECK(cudaEventCreateWithFlags(&fp.join[k], cudaEventDisableTiming));
        }
        SHERRY_CUDA_CHECK(cudaEventCreateWithFlags(&fp.fork, cudaEventDisableTiming));
        fp.ready = true;
    }
    *out = &fp;
    return SHERRY_OK;
}

static int check_shape(int64_t N, int64_t K) {
    if (N < 0 || K < 32 || K > SHERRY_MAX_K || (K % 32) != 0) return SHERRY_ERR_SHAPE;
    if (N > (int64_t)0x7fffffff) return SHERRY_ERR_SHAPE;
    return SHERRY_OK;
}

static int check_gran(int64_t K, int granularity, int group) {
    if (granularity == SHERRY_PER_TENSOR || granularity == SHERRY_PER_CHANNEL) return SHERRY_OK;
    if (granularity != SHERRY_PER_GROUP) return SHERRY_ERR_GRANULARITY;
    if (group <= 0 || (group % 32) != 0 || (K % group) != 0) return SHERRY_ERR_GROUP;
    return SHERRY_OK;
}

static int check_planes(const uint32_t* idx, const uint8_t* sgn, const float* scales, int64_t N) {
    if (N > 0 && (!idx || !sgn || !scales)) return SHERRY_ERR_NULL;
    if (!aligned(idx, 16) || !aligned(sgn, 16) || !aligned(scales, 16)) return SHERRY_ERR_ALIGN;
    return SHERRY_OK;
}

// Which kernel computes each problem of a call.  Problems with one or two tokens
// that fit the streaming lookup-table kernel share one launch of it, problems with
// three to sixteen tokens of the same shapes one launch of its tensor-core form
// (unless their row blocks would outnumber its tickets); 2 <= M <= 8 problems with K % 128 == 0
// share one launch of the warp-MMA kernel; other problems with up to 32 tokens
// that fit the tcgen05 few-token kernel share one launch of it; each problem with
// M >= 17 that fits the prefill kernel gets a launch of its own; what remains
// shares one launch of the general lookup-table kernel.
struct Routes {
    std::vector<ProbShape> stream_s, mstream_s, hmma_s, skinny_s, rest_s;
    std::vector<sherry_linear_desc> stream_d, mstream_d, hmma_d, skinny_d, rest_d;
    std::vector<int> prefill;  // indices into the call's problems
};

static void route(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, Routes& r) {
    int64_t tiles = 0;
    for (int i = 0; i < count; ++i)
        if (stream_eligible(shapes[i], M) || mstream_eligible(shapes[i], M)) tiles += stream_tiles(shapes[i]);
    const bool stream_ok = tiles > 0 && tiles <= kMaxTickets;
    for (int i = 0; i < count; ++i) {
        if (stream_ok && stream_eligible(shapes[i], M)) {
            r.stream_s.push_back(shapes[i]);
            if (descs) r.stream_d.push_back(descs[i]);
        } else if (stream_ok && mstream_eligible(shapes[i], M)) {
            r.mstream_s.push_back(shapes[i]);
            if (descs) r.mstream_d.push_back(descs[i]);
        } else if (hmma_eligible(shapes[i], M)) {
            r.hmma_s.push_back(shapes[i]);
            if (descs) r.hmma_d.push_back(descs[i]);
        } else if (skinny_eligible(shapes[i], M)) {
            r.skinny_s.push_back(shapes[i]);
            if (descs) r.skinny_d.push_back(descs[i]);
        } else if (prefill_eligible(shapes[i], M)) {
            r.prefill.push_back(i);
        } else {
            r.rest_s.push_back(shapes[i]);
            if (descs) r.rest_d.push_back(descs[i]);
        }
    }
}

// The streaming and general lookup-table launches of a call run one after the
// other on its stream and share the workspace (tickets first, both leave them zero).
static size_t linear_ws_bytes(const ProbShape* shapes, int count, int64_t M, int sms) {
    Routes r;
    route(shapes, nullptr, count, M, r);
    size_t ws = 0;
    if (!r.stream_s.empty()) ws = stream_workspace_bytes(r.stream_s.data(), (int)r.stream_s.size(), M, sms);
    if (!r.mstream_s.empty())
        ws = std::max(ws, stream_workspace_bytes(r.mstream_s.data(), (int)r.mstream_s.size(), M, sms));
    if (!r.rest_s.empty()) ws = std::max(ws, lut_workspace_bytes(r.rest_s.data(), (int)r.rest_s.size(), M, sms));
    return ws;
}

static int linear_launch(const ProbShape* shapes, const sherry_linear_desc* descs, int count, int64_t M, int y_bf16,
                         void* workspace, int sms, cudaStream_t stream) {
    Routes r;
    route(shapes, descs, count, M, r);
    int st = SHERRY_OK;
    if (!r.hmma_s.empty() &&
        (st = hmma_linear_launch(r.hmma_s.data(), r.hmma_d.data(), (int)r.hmma_s.size(), M, y_bf16, stream)))
        return st;
    if (!r.skinny_s.empty() &&
        (st = skinny_linear_launch(r.skinny_s.data(), r.skinny_d.data(), (int)r.skinny_s.size(), M, y_bf16, sms,
                                   stream)))
        return st;
    if (r.prefill.size() == 1) {
        if ((st = prefill_launch(shapes[r.prefill[0]], descs[r.prefill[0]], M, y_bf16, stream))) return st;
    } else if (!r.prefill.empty()) {
        std::lock_guard<std::mutex> lk(g_fork_mu);
        ForkPool* fp = nullptr;
        if ((st = fork_pool(&fp))) return st;
        const int ns = std::min(kForkStreams, (int)r.prefill.size());
        SHERRY_CUDA_CHECK(cudaEventRecord(fp->fork, stream));
        for (int k = 0; k < ns; ++k) SHERRY_CUDA_CHECK(cudaStreamWaitEvent(fp->s[k], fp->fork, 0));
        for (size_t j = 0; j < r.prefill.size() && st == SHERRY_OK; ++j) {
            const int i = r.prefill[j];
            st = prefill_launch(shapes[i], descs[i], M, y_bf16, fp->s[j % ns]);
        }
        // joined even after a failed launch, so the caller's stream stays ordered
        for (int k = 0; k < ns; ++k) {
            SHERRY_CUDA_CHECK(cudaEventRecord(fp->join[k], fp->s[k]));
            SHERRY_CUDA_CHECK(cudaStreamWaitEvent(stream, fp->join[k], 0));
        }
        if (st) return st;
    }
    if (!r.stream_s.empty() &&
        (st = stream_linear_launch(r.stream_s.data(), r.stream_d.data(), (int)r.stream_s.size(), M, y_bf16, workspace,
                                   sms, stream)))
        return st;
    if (!r.mstream_s.empty() &&
        (st = mstream_linear_launch(r.mstream_s.data(), r.mstream_d.data(), (int)r.mstream_s.size(), M, y_bf16,
                                    workspace, sms, stream)))
        return st;
    if (r.rest_s.empty()) return SHERRY_OK;
    return lut_linear_launch(r.rest_s.data(), r.rest_d.data(), (int)r.rest_s.size(), M, y_bf16, workspace, sms, stream);
}

}  // namespace sherry

using namespace sherry;

extern "C" {

int sherry_version(void) { return 0x000100; }

int sherry_last_cuda_error(void) { return g_last_cuda_error; }

static std::atomic<int64_t> g_timeouts_seen{0};

int sherry_device_status(void* stream) {
    const int st = device_status_take(static_cast<cudaStream_t>(stream));
    if (st) g_timeouts_seen.fetch_add(1);
    return st;
}

int64_t sherry_timeout_count(void) { return g_timeouts_seen.load(); }

int64_t sherry_set_wait_budget(int64_t cycles) { return (int64_t)stream_set_wait_cycles((long long)cycles); }

const char* sherry_status_string(int status) {
    switch (status) {
        case SHERRY_OK: return "ok";
        case SHERRY_ERR_NULL: return "a required pointer is NULL";
        case SHERRY_ERR_SHAPE: return "bad shape (need N >= 0, M >= 0, 32 <= K <= SHERRY_MAX_K, K % 32 == 0)";
        case SHERRY_ERR_GRANULARITY: return "unknown granularity";
        case SHERRY_ERR_GROUP: return "bad group size (need group > 0, group % 32 == 0, K % group == 0)";
        case SHERRY_ERR_DTYPE: return "unknown element type";
        case SHERRY_ERR_ALIGN: return "misaligned pointer (16-byte alignment required)";
        case SHERRY_ERR_WORKSPACE: return "workspace missing or too small";
        case SHERRY_ERR_CUDA: return "CUDA error (see sherry_last_cuda_error)";
        case SHERRY_ERR_TIMEOUT: return "a bounded device wait gave up";
        case SHERRY_ERR_UNSUPPORTED: return "unsupported on this device or build";
        default: return "unknown status";
    }
}

size_t sherry_idx_bytes(int64_t N, int64_t K) {
    if (check_shape(N, K)) return 0;
    return (size_t)(N * (K / 32)) * 4;
}

size_t sherry_sgn_bytes(int64_t N, int64_t K) {
    if (check_shape(N, K)) return 0;
    return (size_t)(N * (K / 32));
}

int64_t sherry_num_scales(int64_t N, int64_t K, int granularity, int group) {
    if (check_shape(N, K) || check_gran(K, granularity, group)) return -1;
    if (granularity == SHERRY_PER_TENSOR) return 1;
    if (granularity == SHERRY_PER_CHANNEL) return N;
    return N * (K / group);
}

size_t sherry_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int granularity, int group) {
    if (check_shape(N, K) || check_gran(K, granularity, group)) return 0;
    if (op == SHERRY_OP_QUANTIZE_PACK) return quantize_workspace_bytes(N, K, granularity);
    if (op == SHERRY_OP_LINEAR) {
        if (M <= 0 || N == 0) return 0;
        ProbShape s{N, K, granularity, group};
        return linear_ws_bytes(&s, 1, M, device_sms());
    }
    return 0;
}

static int check_quantize_desc(const sherry_quantize_desc& d) {
    int st = check_shape(d.N, d.K);
    if (st) return st;
    if ((st = check_gran(d.K, d.granularity, d.group))) return st;
    if (d.w_dtype != SHERRY_F32 && d.w_dtype != SHERRY_BF16) return SHERRY_ERR_DTYPE;
    if (d.Wq && d.wq_dtype != SHERRY_F32 && d.wq_dtype != SHERRY_BF16) return SHERRY_ERR_DTYPE;
    if (!d.scales || (d.N > 0 && (!d.W || !d.idx || !d.sgn))) return SHERRY_ERR_NULL;
    if (!aligned(d.W, 16) || !aligned(d.idx, 16) || !aligned(d.sgn, 16) || !aligned(d.scales, 16) ||
        !aligned(d.Wq, 16))
        return SHERRY_ERR_ALIGN;
    return SHERRY_OK;
}

static QuantizeJob job_of(const sherry_quantize_desc& d) {
    return QuantizeJob{d.W, d.w_dtype, d.N, d.K, d.granularity, d.group, d.idx, d.sgn, d.scales, d.Wq, d.wq_dtype,
                       nullptr, nullptr, 0.0f};
}

static int quantize_call(const sherry_quantize_desc* descs, int count, void* workspace, size_t workspace_bytes,
                         void* stream) {
    if (!descs && count > 0) return SHERRY_ERR_NULL;
    if (count < 0 || count > SHERRY_MAX_BATCH) return SHERRY_ERR_SHAPE;
    std::vector<QuantizeJob> jobs;
    for (int i = 0; i < count; ++i) {
        const int st = check_quantize_desc(descs[i]);
        if (st) return st;
        jobs.push_back(job_of(descs[i]));
    }
    const size_t need = quantize_batch_workspace_bytes(jobs.data(), count);
    if (need > 0 && (!workspace || workspace_bytes < need)) return SHERRY_ERR_WORKSPACE;
    if (need > 0 && !aligned(workspace, 256)) return SHERRY_ERR_ALIGN;
    if (count == 0) return SHERRY_OK;
    return quantize_jobs_launch(jobs.data(), count, workspace, device_sms(), static_cast<cudaStream_t>(stream));
}

int sherry_quantize_pack(const void* W, int w_dtype, int64_t N, int64_t K, int granularity, int group,
                         uint32_t* idx, uint8_t* sgn, float* scales, void* workspace, size_t workspace_bytes,
                         void* stream) {
    const sherry_quantize_desc d{W, idx, sgn, scales, nullptr, N, K, w_dtype, granularity, group, SHERRY_F32};
    return quantize_call(&d, 1, workspace, workspace_bytes, stream);
}

int sherry_fake_quant(const void* W, int w_dtype, int64_t N, int64_t K, int granularity, int group, void* Wq,
                      int wq_dtype, uint32_t* idx, uint8_t* sgn, float* scales, void* workspace,
                      size_t workspace_bytes, void* stream) {
    if (N > 0 && !Wq) return SHERRY_ERR_NULL;
    const sherry_quantize_desc d{W, idx, sgn, scales, Wq, N, K, w_dtype, granularity, group, wq_dtype};
    return quantize_call(&d, 1, workspace, workspace_bytes, stream);
}

int sherry_quantize_pack_tequila(const void* W, int w_dtype, int64_t N, int64_t K, int granularity, int group,
                                 float eps, uint32_t* idx, uint8_t* sgn, float* scales, uint16_t* D, float* bias,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    const sherry_quantize_desc d{W, idx, sgn, scales, nullptr, N, K, w_dtype, granularity, group, SHERRY_F32};
    int st = check_quantize_desc(d);
    if (st) return st;
    if (N > 0 && !D) return SHERRY_ERR_NULL;
    if (!aligned(D, 16) || !aligned(bias, 4)) return SHERRY_ERR_ALIGN;
    QuantizeJob j = job_of(d);
    j.D = D;
    j.bias = bias;
    j.eps = eps;
    const size_t need = quantize_batch_workspace_bytes(&j, 1);
    if (need > 0 && (!workspace || workspace_bytes < need)) return SHERRY_ERR_WORKSPACE;
    if (need > 0 && !aligned(workspace, 256)) return SHERRY_ERR_ALIGN;
    return quantize_jobs_launch(&j, 1, workspace, device_sms(), static_cast<cudaStream_t>(stream));
}

int sherry_quantize_pack_batched(const sherry_quantize_desc* descs, int count, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    return quantize_call(descs, count, workspace, workspace_bytes, stream);
}

size_t sherry_quantize_pack_batched_workspace_bytes(const sherry_quantize_desc* descs, int count) {
    if (!descs || count <= 0 || count > SHERRY_MAX_BATCH) return 0;
    std::vector<QuantizeJob> jobs;
    for (int i = 0; i < count; ++i) {
        if (check_quantize_desc(descs[i])) return 0;
        jobs.push_back(job_of(descs[i]));
    }
    return quantize_batch_workspace_bytes(jobs.data(), count);
}

static int check_unpack_desc(const sherry_unpack_desc& d) {
    int st = check_shape(d.N, d.K);
    if (st) return st;
    if ((st = check_gran(d.K, d.granularity, d.group))) return st;
    if ((st = check_planes(d.idx, d.sgn, d.scales, d.N))) return st;
    if (d.N > 0 && !d.W_out) return SHERRY_ERR_NULL;
    if (!aligned(d.W_out, 16)) return SHERRY_ERR_ALIGN;
    return SHERRY_OK;
}

int sherry_unpack(const uint32_t* idx, const uint8_t* sgn, const float* scales, int64_t N, int64_t K,
                  int granularity, int group, uint16_t* W_out, void* stream) {
    const sherry_unpack_desc d{idx, sgn, scales, N, K, granularity, group, W_out};
    const int st = check_unpack_desc(d);
    if (st) return st;
    return unpack_launch(&d, 1, static_cast<cudaStream_t>(stream), device_sms());
}

int sherry_unpack_batched(const sherry_unpack_desc* descs, int count, void* stream) {
    if (!descs && count > 0) return SHERRY_ERR_NULL;
    if (count < 0 || count > SHERRY_MAX_BATCH) return SHERRY_ERR_SHAPE;
    for (int i = 0; i < count; ++i) {
        const int st = check_unpack_desc(descs[i]);
        if (st) return st;
    }
    if (count == 0) return SHERRY_OK;
    return unpack_launch(descs, count, static_cast<cudaStream_t>(stream), device_sms());
}

static int check_linear_desc(const sherry_linear_desc& d, int64_t M) {
    int st = check_shape(d.N, d.K);
    if (st) return st;
    if ((st = check_gran(d.K, d.granularity, d.group))) return st;
    if ((st = check_planes(d.idx, d.sgn, d.scales, d.N))) return st;
    if (M > 0 && d.N > 0 && (!d.X || !d.Y)) return SHERRY_ERR_NULL;
    if (!aligned(d.X, 16) || !aligned(d.Y, 16)) return SHERRY_ERR_ALIGN;
    return SHERRY_OK;
}

int sherry_linear(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* idx, const uint8_t* sgn,
                  const float* scales, int granularity, int group, void* Y, int y_dtype, void* workspace,
                  size_t workspace_bytes, void* stream) {
    if (M < 0 || M > (int64_t)0x7fffffff) return SHERRY_ERR_SHAPE;
    sherry_linear_desc d{X, idx, sgn, scales, Y, N, K, granularity, group};
    int st = check_linear_desc(d, M);
    if (st) return st;
    if (y_dtype != SHERRY_F32 && y_dtype != SHERRY_BF16) return SHERRY_ERR_DTYPE;
    if (M == 0 || N == 0) return SHERRY_OK;
    ProbShape s{N, K, granularity, group};
    const int sms = device_sms();
    const size_t need = linear_ws_bytes(&s, 1, M, sms);
    if (need > 0 && (!workspace || workspace_bytes < need)) return SHERRY_ERR_WORKSPACE;
    if (need > 0 && !aligned(workspace, 256)) return SHERRY_ERR_ALIGN;
    return linear_launch(&s, &d, 1, M, y_dtype == SHERRY_BF16, workspace, sms, static_cast<cudaStream_t>(stream));
}

static int batch_shapes(const sherry_linear_desc* descs, int count, int64_t M, std::vector<ProbShape>& shapes,
                        std::vector<sherry_linear_desc>& kept) {
    if (!descs && count > 0) return SHERRY_ERR_NULL;
    if (count < 0 || count > SHERRY_MAX_BATCH) return SHERRY_ERR_SHAPE;
    if (M < 0 || M > (int64_t)0x7fffffff) return SHERRY_ERR_SHAPE;
    for (int i = 0; i < count; ++i) {
        int st = check_linear_desc(descs[i], M);
        if (st) return st;
        if (descs[i].N == 0) continue;
        shapes.push_back(ProbShape{descs[i].N, descs[i].K, descs[i].granularity, descs[i].group});
        kept.push_back(descs[i]);
    }
    return SHERRY_OK;
}

size_t sherry_linear_batched_workspace_bytes(const sherry_linear_desc* descs, int count, int64_t M) {
    std::vector<ProbShape> shapes;
    std::vector<sherry_linear_desc> kept;
    if (batch_shapes(descs, count, M, shapes, kept) || shapes.empty() || M == 0) return 0;
    return linear_ws_bytes(shapes.data(), (int)shapes.size(), M, device_sms());
}

int sherry_linear_batched(const sherry_linear_desc* descs, int count, int64_t M, int y_dtype, void* workspace,
                          size_t workspace_bytes, void* stream) {
    std::vector<ProbShape> shapes;
    std::vector<sherry_linear_desc> kept;
    int st = batch_shapes(descs, count, M, shapes, kept);
    if (st) return st;
    if (y_dtype != SHERRY_F32 && y_dtype != SHERRY_BF16) return SHERRY_ERR_DTYPE;
    if (shapes.empty() || M == 0) return SHERRY_OK;
    const int sms = device_sms();
    const size_t need = linear_ws_bytes(shapes.data(), (int)shapes.size(), M, sms);
    if (need > 0 && (!workspace || workspace_bytes < need)) return SHERRY_ERR_WORKSPACE;
    if (need > 0 && !aligned(workspace, 256)) return SHERRY_ERR_ALIGN;
    return linear_launch(shapes.data(), kept.data(), (int)shapes.size(), M, y_dtype == SHERRY_BF16, workspace, sms,
                         static_cast<cudaStream_t>(stream));
}

// The Tequila-style linear: the packed linear into fp32 (Y itself, or scratch after
// the linear's workspace for bf16 Y), then the dead-weight term.  The fp32 scratch
// never overlaps the ticket region at the front of the workspace, even when the
// linear itself needs no workspace: other linear calls sharing the buffer rely on
// that region being zero.
static size_t tequila_ws(int64_t M, int64_t N, int64_t K, int granularity, int group, int y_dtype, size_t* lin_ws) {
    ProbShape s{N, K, granularity, group};
    const size_t lw = linear_ws_bytes(&s, 1, M, device_sms());
    *lin_ws = (lw + 255) & ~(size_t)255;
    if (y_dtype != SHERRY_BF16) return lw;
    *lin_ws = std::max(*lin_ws, kTicketBytes);
    return *lin_ws + (size_t)(M * N) * sizeof(float);
}

size_t sherry_linear_tequila_workspace_bytes(int64_t M, int64_t N, int64_t K, int granularity, int group,
                                             int y_dtype) {
    if (check_shape(N, K) || check_gran(K, granularity, group) || M <= 0 || N == 0) return 0;
    size_t lw = 0;
    return tequila_ws(M, N, K, granularity, group, y_dtype, &lw);
}

int sherry_linear_tequila(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* idx, const uint8_t* sgn,
                          const float* scales, int granularity, int group, const uint16_t* D, const float* bias,
                          int mode, void* Y, int y_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    if (M < 0 || M > (int64_t)0x7fffffff) return SHERRY_ERR_SHAPE;
    sherry_linear_desc d{X, idx, sgn, scales, Y, N, K, granularity, group};
    int st = check_linear_desc(d, M);
    if (st) return st;
    if (y_dtype != SHERRY_F32 && y_dtype != SHERRY_BF16) return SHERRY_ERR_DTYPE;
    if (mode != SHERRY_TEQUILA_ONES && mode != SHERRY_TEQUILA_SIGN) return SHERRY_ERR_SHAPE;
    if (M > 0 && N > 0 && ((mode == SHERRY_TEQUILA_ONES && !bias) || (mode == SHERRY_TEQUILA_SIGN && !D)))
        return SHERRY_ERR_NULL;
    if (!aligned(D, 16) || !aligned(bias, 4)) return SHERRY_ERR_ALIGN;
    if (M == 0 || N == 0) return SHERRY_OK;
    size_t lw = 0;
    const size_t need = tequila_ws(M, N, K, granularity, group, y_dtype, &lw);
    if (need > 0 && (!workspace || workspace_bytes < need)) return SHERRY_ERR_WORKSPACE;
    if (need > 0 && !aligned(workspace, 256)) return SHERRY_ERR_ALIGN;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* y32 = y_dtype == SHERRY_BF16 ? reinterpret_cast<float*>(static_cast<char*>(workspace) + lw)
                                        : static_cast<float*>(Y);
    ProbShape ps{N, K, granularity, group};
    d.Y = y32;
    if ((st = linear_launch(&ps, &d, 1, M, 0, workspace, device_sms(), s))) return st;
    return tequila_term_launch(X, M, N, K, idx, D, bias, mode, y32, Y, y_dtype == SHERRY_BF16, s);
}

int sherry_arenas_linear(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* idx, const uint8_t* sgn,
                         const float* scales, int granularity, int group, const uint16_t* Wd, float lambda, void* Y,
                         int y_dtype, void* stream) {
    if (M < 0 || M > (int64_t)0x7fffffff) return SHERRY_ERR_SHAPE;
    const sherry_linear_desc d{X, idx, sgn, scales, Y, N, K, granularity, group};
    int st = check_linear_desc(d, M);
    if (st) return st;
    if (y_dtype != SHERRY_F32 && y_dtype != SHERRY_BF16) return SHERRY_ERR_DTYPE;
    if (M > 0 && N > 0 && !Wd) return SHERRY_ERR_NULL;
    if (!aligned(Wd, 16)) return SHERRY_ERR_ALIGN;
    if (M == 0 || N == 0) return SHERRY_OK;
    const ProbShape s{N, K, granularity, group};
    if (!arenas_eligible(s, M)) return SHERRY_ERR_UNSUPPORTED;
    return arenas_launch(s, d, M, y_dtype == SHERRY_BF16, Wd, lambda, static_cast<cudaStream_t>(stream));
}

float sherry_arenas_lambda(int64_t step, int64_t total, float lambda0) {
    if (total <= 0) return lambda0;
    const double t = (double)(step < 0 ? 0 : (step > total ? total : step));
    return (float)((double)lambda0 * 0.5 * (1.0 + cos(3.14159265358979323846 * t / (double)total)));
}

// A chain without its empty linears: problems, descriptors and phase bounds.
struct Chain {
    std::vector<ProbShape> shapes;
    std::vector<sherry_linear_desc> descs;
    std::vector<int> begin;  // n_phases + 1 problem indices
};

static int chain_of(const sherry_linear_desc* descs, int count, const int* phase_begin, int n_phases, int64_t M,
                    Chain& c) {
    if ((!descs && count > 0) || !phase_begin) return SHERRY_ERR_NULL;
    if (count < 0 || count > SHERRY_MAX_BATCH || n_phases < 1 || n_phases > SHERRY_MAX_BATCH) return SHERRY_ERR_SHAPE;
    if (M < 0 || M > (int64_t)0x7fffffff) return SHERRY_ERR_SHAPE;
    if (phase_begin[0] != 0 || phase_begin[n_phases] != count) return SHERRY_ERR_SHAPE;
    for (int ph = 0; ph < n_phases; ++ph)
        if (phase_begin[ph + 1] < phase_begin[ph]) return SHERRY_ERR_SHAPE;
    for (int ph = 0; ph < n_phases; ++ph) {
        c.begin.push_back((int)c.shapes.size());
        for (int i = phase_begin[ph]; i < phase_begin[ph + 1]; ++i) {
            const int st = check_linear_desc(descs[i], M);
            if (st) return st;
            if (descs[i].N == 0) continue;
            c.shapes.push_back(ProbShape{descs[i].N, descs[i].K, descs[i].granularity, descs[i].group});
            c.descs.push_back(descs[i]);
        }
    }
    c.begin.push_back((int)c.shapes.size());
    return SHERRY_OK;
}

static size_t chain_ws(const Chain& c, int64_t M, int sms) {
    const int n = (int)c.begin.size() - 1;
    if (c.shapes.empty() || M == 0) return 0;
    if (chain_launch_ok(c.shapes.data(), (int)c.shapes.size(), n, M))
        return chain_workspace_bytes(c.shapes.data(), (int)c.shapes.size(), c.begin.data(), n, M, sms);
    size_t ws = 0;
    for (int ph = 0; ph < n; ++ph)
        if (c.begin[ph + 1] > c.begin[ph])
            ws = std::max(ws, linear_ws_bytes(c.shapes.data() + c.begin[ph], c.begin[ph + 1] - c.begin[ph], M, sms));
    return ws;
}

size_t sherry_linear_chain_workspace_bytes(const sherry_linear_desc* descs, int count, const int* phase_begin,
                                           int n_phases, int64_t M) {
    Chain c;
    if (chain_of(descs, count, phase_begin, n_phases, M, c)) return 0;
    return chain_ws(c, M, device_sms());
}

int sherry_linear_chain(const sherry_linear_desc* descs, int count, const int* phase_begin, int n_phases, int64_t M,
                        int y_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    Chain c;
    int st = chain_of(descs, count, phase_begin, n_phases, M, c);
    if (st) return st;
    if (y_dtype != SHERRY_F32 && y_dtype != SHERRY_BF16) return SHERRY_ERR_DTYPE;
    if (c.shapes.empty() || M == 0) return SHERRY_OK;
    const int sms = device_sms();
    const size_t need = chain_ws(c, M, sms);
    if (need > 0 && (!workspace || workspace_bytes < need)) return SHERRY_ERR_WORKSPACE;
    if (need > 0 && !aligned(workspace, 256)) return SHERRY_ERR_ALIGN;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int n = (int)c.begin.size() - 1;
    if (chain_launch_ok(c.shapes.data(), (int)c.shapes.size(), n, M))
        return chain_linear_launch(c.shapes.data(), c.descs.data(), (int)c.shapes.size(), c.begin.data(), n, M,
                                   y_dtype == SHERRY_BF16, workspace, sms, s);
    // otherwise one batched launch set per phase, ordered by the stream
    for (int ph = 0; ph < n; ++ph) {
        const int b = c.begin[ph], e = c.begin[ph + 1];
        if (e > b && (st = linear_launch(c.shapes.data() + b, c.descs.data() + b, e - b, M, y_dtype == SHERRY_BF16,
                                         workspace, sms, s)))
            return st;
    }
    return SHERRY_OK;
}

}  // extern "C"
