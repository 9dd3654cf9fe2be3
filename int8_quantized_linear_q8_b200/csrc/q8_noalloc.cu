// q8_noalloc.cu -- q8_linear_w8a8 for callers that cannot allocate device memory.
//
// q8_linear_w8a8 needs scratch for the activation codes it computes before the integer
// matmul, and asks its caller for that scratch as a workspace.  Some callers cannot
// provide one: a host runtime that has reserved all device memory for its own pool, a
// latency-critical loop in which cudaMalloc's implicit device-wide synchronisation is not
// acceptable, or a bare C caller with no allocator of its own.  q8_linear_w8a8_noalloc
// serves them with a fixed scratch array that is part of the library image itself, so
// neither the library nor the caller allocates anything per call.
//
// The array below is an ordinary module-scope device variable: each GPU on which the
// library's device code is loaded holds its kNoAllocScratchBytes until the process exits.
// In host code its name stands for a host-side shadow, not a device address, so the
// entry point looks up the real device address once per device (cudaGetSymbolAddress,
// with that device current) and passes that pointer down as the workspace.
#include "q8_kernels.cuh"

#include <mutex>

namespace q8 {

// Largest scratch q8_linear_w8a8_noalloc can use: M*K bytes of codes for one pass, twice
// that for two passes (each rounded up to 256 bytes).  16 MiB covers, for example,
// M = 4096 x K = 4096 with one pass or M = 2048 x K = 960 with two.
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;

static __device__ __align__(256) int8_t g_noalloc_scratch[kNoAllocScratchBytes];

static void* g_noalloc_ptr[128];
static bool g_noalloc_ready[128];
static std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, looked up on the first call
// made with that device current and remembered afterwards.
static q8_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    if (dev < 0 || dev >= 128) return Q8_ERR_UNSUPPORTED_ARCH;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ready[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return Q8_ERR_LAUNCH;
        }
        g_noalloc_ptr[dev] = p;
        g_noalloc_ready[dev] = true;
    }
    *out = g_noalloc_ptr[dev];
    return Q8_OK;
}

}  // namespace q8

extern "C" q8_status q8_linear_w8a8_noalloc(const float* x, q8_qparams first,
                                            const q8_qparams* second, const int8_t* q,
                                            const int32_t* wsum, const float* s_w, float* y,
                                            int64_t M, int64_t N, int64_t K, void* stream) {
    // The same argument checks, in the same order, as q8_linear_w8a8 (so both report the
    // same status for the same mistake), then the device, then the built-in size limit.
    q8_status st = q8::w8a8_check_args(x, first, second, q, wsum, s_w, nullptr, y, M, N, K);
    if (st != Q8_OK || M == 0) return st;
    st = q8::check_current_device();
    if (st != Q8_OK) return st;
    const size_t need =
        q8_workspace_bytes(Q8_OP_LINEAR_W8A8, M, N, K, second != nullptr ? 1 : 0);
    if (need > q8::kNoAllocScratchBytes) return Q8_ERR_WORKSPACE;
    void* scratch = nullptr;
    st = q8::noalloc_scratch(&scratch);
    if (st != Q8_OK) return st;
    // Every step after this is q8_linear_w8a8 itself, with the built-in array as workspace.
    return q8_linear_w8a8(x, first, second, q, wsum, s_w, y, M, N, K, scratch,
                          q8::kNoAllocScratchBytes, stream);
}
