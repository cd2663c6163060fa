// noalloc.cu -- sherry_linear_noalloc: the packed linear without a caller
// workspace, for callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not an option -- inside a
// region whose memory was planned ahead by a host framework that hands out no
// scratch buffers, in plugins that only receive input and output pointers, or
// in latency-critical paths that must not enter the allocator.  This entry
// point takes the same arguments as sherry_linear minus the workspace.
//
// Its scratch (split-K tickets and partial sums) lives in one file-scope device
// array of fixed size, loaded with the library and held by every GPU that
// loads it until the process exits.  All calls share that array, so calls that
// overlap on the GPU (different streams, different host threads) race; keep
// them ordered on one stream.  Each call zeroes the ticket region before its
// kernel, so a call never depends on what an earlier call left behind.
#include "common.cuh"

#include <mutex>
#include <vector>

namespace sherry {

constexpr size_t kNoallocBytes = SHERRY_NOALLOC_SCRATCH_BYTES;  // 256 KiB of tickets, then partial sums
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocBytes];

// Device address of the array for the current device, looked up once per device
// with that device current (host code cannot use the symbol as an address).
static int noalloc_scratch(void** out) {
    static std::mutex mu;
    static std::vector<void*> ptrs;
    int dev = 0;
    SHERRY_CUDA_CHECK(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lk(mu);
    if ((int)ptrs.size() <= dev) ptrs.resize(dev + 1, nullptr);
    if (!ptrs[dev]) {
        void* p = nullptr;
        SHERRY_CUDA_CHECK(cudaGetSymbolAddress(&p, g_noalloc_scratch));
        ptrs[dev] = p;
    }
    *out = ptrs[dev];
    return SHERRY_OK;
}

}  // namespace sherry

using namespace sherry;

extern "C" int sherry_linear_noalloc(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* idx,
                                     const uint8_t* sgn, const float* scales, int granularity, int group, void* Y,
                                     int y_dtype, void* stream) {
    // how much scratch the ordinary call would ask for (0 on invalid arguments,
    // which sherry_linear then reports)
    const size_t need = sherry_workspace_bytes(SHERRY_OP_LINEAR, M, N, K, granularity, group);
    if (need > kNoallocBytes) return SHERRY_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0) {
        int st = noalloc_scratch(&ws);
        if (st) return st;
        // tickets must start at zero: clear the ticket region on this stream
        SHERRY_CUDA_CHECK(cudaMemsetAsync(ws, 0, kTicketBytes, static_cast<cudaStream_t>(stream)));
    }
    return sherry_linear(X, M, N, K, idx, sgn, scales, granularity, group, Y, y_dtype, ws, need, stream);
}
