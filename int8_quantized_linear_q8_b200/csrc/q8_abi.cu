// q8_abi.cu -- the C ABI (include/q8.h): argument checks on the host, then kernel
// launches on the caller's stream.  Nothing here allocates device memory, synchronises
// (except q8_last_device_status, documented as synchronising) or aborts.
#include "q8_kernels.cuh"

#include <float.h>
#include <math.h>
#include <mutex>

namespace q8 {

// Status word that kernels with bounded waits set when a wait expires (0 = none).
// Kernels receive its device address as an argument (kernels live in other files).
__device__ int g_device_status;

static q8_status read_and_clear_device_status() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    if (v == 0) return Q8_OK;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return Q8_ERR_DEVICE;
}

// ------------------------------------------------------------------- device checks
struct DevInfo {
    int checked = 0;
    int ok = 0;
    int num_sms = 0;
    int* status = nullptr;     // device address of g_device_status on this device
};
static DevInfo g_dev[128];
static std::mutex g_dev_mu;

static q8_status current_device(int& num_sms, int** status = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    if (dev < 0 || dev >= 128) return Q8_ERR_UNSUPPORTED_ARCH;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DevInfo& d = g_dev[dev];
    if (!d.checked) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return Q8_ERR_LAUNCH;
        }
        d.ok = (major == 10 && minor == 0);
        d.num_sms = sms;
        if (d.ok) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
                cudaGetLastError();
                return Q8_ERR_LAUNCH;
            }
            d.status = static_cast<int*>(p);
        }
        d.checked = 1;
    }
    num_sms = d.num_sms;
    if (status) *status = d.status;
    return d.ok ? Q8_OK : Q8_ERR_UNSUPPORTED_ARCH;
}

static inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
static inline bool aligned4(const void* p) { return ((uintptr_t)p & 3u) == 0; }

static inline q8_status check_k(int64_t K) {
    if (K < 16 || K > 65535 || (K % 16) != 0) return Q8_ERR_SHAPE;
    return Q8_OK;
}

static inline q8_status check_qparams(const q8_qparams& p) {
    if (!(p.scale > 0.0f) || !isfinite(p.scale)) return Q8_ERR_ARG;
    if (p.zero_point < -128 || p.zero_point > 127) return Q8_ERR_ARG;
    return Q8_OK;
}

static inline q8_status launched(cudaError_t e) {
    if (e != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return Q8_OK;
}

#define Q8_TRY(expr)                      \
    do {                                  \
        q8_status _s = (expr);            \
        if (_s != Q8_OK) return _s;       \
    } while (0)

static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Host-side checks of the W8A8 linear's arguments other than the workspace (shared by the
// workspace and the allocation-free entry points, so both report the same status codes).
q8_status w8a8_check_args(const float* x, const q8_qparams& first, const q8_qparams* second,
                          const int8_t* q, const int32_t* wsum, const float* s_w,
                          const float* bias, const float* y, int64_t M, int64_t N, int64_t K) {
    if (M < 0 || M > 0x7fffffff || N < 1 || N > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    Q8_TRY(check_qparams(first));
    if (second) Q8_TRY(check_qparams(*second));
    if (M == 0) return Q8_OK;
    if (!x || !q || !wsum || !s_w || !y) return Q8_ERR_NULL;
    if (!aligned16(x) || !aligned16(q) || !aligned16(y) || !aligned4(bias)) return Q8_ERR_ALIGN;
    return Q8_OK;
}

// The current device's arch check, for entry points in other files.
q8_status check_current_device() {
    int sms = 0;
    return current_device(sms);
}

// Activation rows up to which the W8A8 linear always runs as a GEMV (weights streamed once
// per 16 rows); above it the tensor-core GEMM takes over, except for small problems: the
// GEMM's fixed cost (quantizer pre-kernel, operand pipeline fill, one tile per CTA) is
// ~8.5 us at K = 960, while the GEMV costs ~4 us plus ~0.55 us per MB of weight it
// streams (measured on B200, K = 960 / 4096, N = 960..4096, M = 32..512), so the GEMV
// keeps problems whose weight passes (ceil(M / 16) x N x K bytes, x 1.6 for two passes)
// stay below 6 MB.  The tensor-core path loads K in 128-byte steps and needs at least one
// whole step.
constexpr int64_t kW8A8GemvMaxM = 16;
constexpr int64_t kW8A8GemvSmallBytes = (int64_t)6 << 20;
constexpr int64_t kTcMinK = 128;
constexpr int64_t kGptqMaxK = 16384;     // three K x K float64 work matrices (6 GB at the cap)

// Workspace plans (byte offsets inside the caller's workspace).  The W8A8 GEMV computes
// its activation codes in registers and needs none; the tensor-core path keeps them in the
// workspace between the quantizer and the GEMM.
static inline bool w8a8_uses_gemv(int64_t M, int64_t N, int64_t K, int two) {
    if (M <= kW8A8GemvMaxM || K < kTcMinK) return true;
    const double passes = (double)((M + 15) / 16) * (double)N * (double)K * (two ? 1.6 : 1.0);
    return passes <= (double)kW8A8GemvSmallBytes;
}
struct W8A8Plan {
    size_t xq1 = 0, xq2 = 0, bytes = 0;
};
static W8A8Plan plan_w8a8(int64_t M, int64_t N, int64_t K, int two) {
    W8A8Plan p;
    if (w8a8_uses_gemv(M, N, K, two)) return p;
    const size_t codes = align_up((size_t)M * (size_t)K, 256);
    p.xq1 = 0;
    p.xq2 = two ? codes : 0;
    p.bytes = M > 0 ? codes * (two ? 2 : 1) : 0;
    return p;
}

// Activation rows up to which the 8da4w linear runs as a GEMV on the packed int4 weights;
// above it a tensor-core GEMM runs: for 17..64 rows the bf16 one that expands the int4
// codes in shared memory (k_q4_gemm_fused); above 64 rows either the int8 one
// (k_q4_gemm_i8: the codes expanded to int8 in shared memory, zero-point term in the
// epilogue) or the bf16 one on a per-call bf16 copy of the weight (k_q4_gemm_tc).
constexpr int64_t kQ4GemvMaxM = 16;

// Above 64 rows: whether the int8 GEMM runs.  Its epilogue converts each group partial
// and applies the zero-point term per element, against the bf16 GEMM's one multiply-add,
// so it pays only with few groups; from 2048 rows the bf16 GEMM uses 256-row activation
// tiles (twice the work per MMA).  Measured at K = 4096, N = 11008, us, bf16 / int8, at
// M = 128, 512, 1024, 2048, 4096:
//   G = 256: 62 / 37, 113 / 65, 169 / 116, 208 / 193, 371 / 344
//   G = 128: 64 / 49, 121 / 90, 182 / 171, 235 / 293, 422 / 534
//   G =  64: 68 / 77, 139 / 144, 210 / 279, 396 / 481, 748 / 883
//   G =  32: 76 / 132, 164 / 254, 251 / 497, 466 / 864, 852 / 1589
static bool q4_use_i8(int64_t M, int G) { return G >= 256 || (G == 128 && M < 2048); }

struct Q4Plan {
    bool tc = false, i8 = false;
    size_t xq = 0, s = 0, z = 0, wb = 0, bytes = 0;
};
// sms: the device's SM count (sizes the K-split workspace of the fused GEMM, 17..64 rows)
static Q4Plan plan_q4(int64_t M, int64_t N, int64_t K, int G, int sms) {
    Q4Plan p;
    if (M <= 0) return p;
    p.tc = M > kQ4GemvMaxM;
    p.i8 = p.tc && !q4_tc_fused(M) && q4_use_i8(M, G);
    // int8 codes [M, K]; for the bf16 GEMMs bf16 (xq - z) [M, K] instead
    const size_t codes = (size_t)M * (size_t)K * (p.tc && !p.i8 ? 2 : 1);
    p.xq = 0;
    p.s = align_up(codes, 256);
    p.z = p.s + align_up((size_t)M * 4, 256);
    p.wb = p.z + align_up((size_t)M * 4, 256);
    // at wb: the int8 GEMM's per-group code sums (fp32 [N, K/G]), or the bf16 copy of the
    // weight, or (17..64 rows) the fused GEMM's K-split partial sums, if it splits
    size_t rest = 0;
    if (p.i8)
        rest = align_up((size_t)N * (size_t)(K / G) * 4, 256);
    else if (p.tc && !q4_tc_fused(M))
        rest = align_up((size_t)N * (size_t)K * 2, 256);
    else if (p.tc)
        rest = align_up(q4_fused_workspace_bytes(M, N, (int)K, G, sms), 256);
    p.bytes = p.wb + rest;
    return p;
}
static inline bool valid_group(int G) { return G == 32 || G == 64 || G == 128 || G == 256; }

// Self-test of the bounded-wait path: one CTA waits on an mbarrier that nothing will ever
// complete, with a short limit; the wait gives up, records kStatusWaitTimeout in the status
// word and the kernel returns normally.
__global__ void k_selftest_bounded_wait(unsigned long long limit_ns, int* status,
                                        int* result) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = mbar_wait_limit(&bar, 0, status, &abort_flag, limit_ns);
    if (threadIdx.x == 0) *result = ok ? 1 : 0;
}

}  // namespace q8

using namespace q8;

extern "C" {

const char* q8_status_string(q8_status s) {
    switch (s) {
        case Q8_OK: return "ok";
        case Q8_ERR_NULL: return "a required pointer is NULL";
        case Q8_ERR_SHAPE: return "a size is out of range";
        case Q8_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case Q8_ERR_ARG: return "invalid argument";
        case Q8_ERR_UNSUPPORTED_ARCH: return "the current device is not sm_100 (B200)";
        case Q8_ERR_LAUNCH: return "a CUDA call failed";
        case Q8_ERR_WORKSPACE: return "workspace missing or too small";
        case Q8_ERR_DEVICE: return "a kernel recorded a device-side failure";
    }
    return "unknown status";
}

int q8_version(void) { return 100; }

q8_status q8_quantize_weight(const float* W, int64_t N, int64_t K, int8_t* q, float* s_w,
                             int32_t* wsum, void* stream) {
    return q8_quantize_weight_grid(W, N, K, Q8_GRID_SYM127, q, s_w, wsum, stream);
}

q8_status q8_quantize_weight_grid(const float* W, int64_t N, int64_t K, q8_grid grid, int8_t* q,
                                  float* s_w, int32_t* wsum, void* stream) {
    if (grid != Q8_GRID_SYM127 && grid != Q8_GRID_FULL128) return Q8_ERR_ARG;
    if (!W || !q || !s_w) return Q8_ERR_NULL;
    if (N < 1 || N > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (!aligned16(W) || !aligned16(q)) return Q8_ERR_ALIGN;
    int sms = 0;
    Q8_TRY(current_device(sms));
    return launched(launch_quantize_weight(W, N, (int)K, grid == Q8_GRID_FULL128 ? 1 : 0, q, s_w,
                                           wsum, (cudaStream_t)stream));
}

q8_status q8_choose_qparams(const void* x, q8_dtype xt, int64_t M, int64_t K, float* s,
                            int32_t* z, int8_t* xq, void* stream) {
    if (xt != Q8_BF16) return Q8_ERR_ARG;
    if (M < 0 || M > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (M == 0) return Q8_OK;
    if (!x || !s || !z) return Q8_ERR_NULL;
    if (!aligned16(x) || (xq && !aligned16(xq))) return Q8_ERR_ALIGN;
    int sms = 0;
    Q8_TRY(current_device(sms));
    return launched(launch_choose_qparams((const uint16_t*)x, M, (int)K, s, z, xq,
                                          (cudaStream_t)stream));
}

q8_status q8_quantize_static(const float* x, int64_t M, int64_t K, q8_qparams first,
                             const q8_qparams* second, int8_t* xq1, int8_t* xq2, void* stream) {
    if (M < 0) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    Q8_TRY(check_qparams(first));
    if (second) Q8_TRY(check_qparams(*second));
    if (M == 0) return Q8_OK;
    if (!x || !xq1 || (second && !xq2)) return Q8_ERR_NULL;
    if (!aligned16(x) || !aligned16(xq1) || (second && !aligned16(xq2))) return Q8_ERR_ALIGN;
    int sms = 0;
    Q8_TRY(current_device(sms));
    return launched(launch_quantize_static(x, M, (int)K, first.scale, first.zero_point,
                                           second != nullptr, second ? second->scale : 1.0f,
                                           second ? second->zero_point : 0, xq1, xq2,
                                           (cudaStream_t)stream, sms));
}

q8_status q8_observe_minmax(const float* x, int64_t n, float* minmax, int reset, void* stream) {
    if (n < 0) return Q8_ERR_SHAPE;
    if (!minmax || (n > 0 && !x)) return Q8_ERR_NULL;
    if (n == 0 && !reset) return Q8_OK;
    if (x && !aligned16(x)) return Q8_ERR_ALIGN;
    int sms = 0;
    Q8_TRY(current_device(sms));
    return launched(
        launch_observe_minmax(x, n, minmax, reset, 0, 1.0f, 0, (cudaStream_t)stream, sms));
}

q8_status q8_observe_residual_minmax(const float* x, int64_t n, q8_qparams first, float* minmax,
                                     int reset, void* stream) {
    if (n < 0) return Q8_ERR_SHAPE;
    Q8_TRY(check_qparams(first));
    if (!minmax || (n > 0 && !x)) return Q8_ERR_NULL;
    if (n == 0 && !reset) return Q8_OK;
    if (x && !aligned16(x)) return Q8_ERR_ALIGN;
    int sms = 0;
    Q8_TRY(current_device(sms));
    return launched(launch_observe_minmax(x, n, minmax, reset, 1, first.scale, first.zero_point,
                                          (cudaStream_t)stream, sms));
}

q8_status q8_qparams_from_minmax(float mn, float mx, q8_qparams* out) {
    if (!out) return Q8_ERR_NULL;
    if (!isfinite(mn) || !isfinite(mx) || mn > mx) return Q8_ERR_ARG;
    // Same formula as the device's per-row rule; plain IEEE fp32 host arithmetic.
    volatile float lo = mn < 0.0f ? mn : 0.0f;
    volatile float hi = mx > 0.0f ? mx : 0.0f;
    volatile float range = hi - lo;
    volatile float s = range / 255.0f;
    if (s < FLT_EPSILON) s = FLT_EPSILON;
    volatile float ratio = lo / s;
    float zf = -128.0f - nearbyintf(ratio);
    if (zf < -128.0f) zf = -128.0f;
    if (zf > 127.0f) zf = 127.0f;
    out->scale = s;
    out->zero_point = (int32_t)zf;
    return Q8_OK;
}

q8_status q8_quantize_weight_q4gs(const float* W, int64_t N, int64_t K, int G, uint8_t* q4,
                                  float* gs, float* c, void* stream) {
    if (!W || !q4 || !gs) return Q8_ERR_NULL;
    if (G != 32 && G != 64 && G != 128 && G != 256) return Q8_ERR_ARG;
    if (N < 1 || N > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (K % G) return Q8_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(q4) || !aligned16(gs) || !aligned4(c)) return Q8_ERR_ALIGN;
    int sms = 0;
    Q8_TRY(current_device(sms));
    cudaStream_t st = (cudaStream_t)stream;
    Q8_TRY(launched(launch_quantize_weight_q4gs(W, N, (int)K, G, q4, gs, st)));
    if (!c) return Q8_OK;
    return launched(launch_q4gs_zero_fold(q4, gs, G, N, (int)K, c, st));
}

q8_status q8_linear_w8a16(const void* x, const int8_t* q, const float* s_w, void* y,
                          q8_dtype yt, int64_t M, int64_t N, int64_t K, void* stream) {
    return q8_linear_w8a16_bias(x, q, s_w, nullptr, y, yt, M, N, K, stream);
}

q8_status q8_linear_w8a16_bias(const void* x, const int8_t* q, const float* s_w,
                               const float* bias, void* y, q8_dtype yt, int64_t M, int64_t N,
                               int64_t K, void* stream) {
    if (yt != Q8_F32 && yt != Q8_BF16) return Q8_ERR_ARG;
    if (M < 0 || M > 0x7fffffff || N < 1 || N > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (M == 0) return Q8_OK;
    if (!x || !q || !s_w || !y) return Q8_ERR_NULL;
    if (!aligned16(x) || !aligned16(q) || !aligned4(bias)) return Q8_ERR_ALIGN;
    int sms = 0;
    int* status = nullptr;
    Q8_TRY(current_device(sms, &status));
    if (w8a16_tma_fits(M, K, bias != nullptr))
        return launched(launch_w8a16_tma((const uint16_t*)x, q, s_w, bias, y, yt == Q8_BF16, M,
                                         N, (int)K, (cudaStream_t)stream, sms, status));
    return launched(launch_w8a16_gemv((const uint16_t*)x, q, s_w, bias, y, yt == Q8_BF16, M, N,
                                      (int)K, (cudaStream_t)stream, sms));
}

size_t q8_workspace_bytes(q8_op op, int64_t M, int64_t N, int64_t K, int extra) {
    if (M < 0 || N < 1 || check_k(K) != Q8_OK) return 0;
    switch (op) {
        case Q8_OP_LINEAR_W8A8: return plan_w8a8(M, N, K, extra != 0).bytes;
        case Q8_OP_GPTQ_INT8:
            if (K > kGptqMaxK || !gptq_block_ok(extra)) return 0;
            return plan_gptq(N, K).bytes;
        case Q8_OP_LINEAR_DQ8CA_Q4GSW: {
            if (!valid_group(extra) || K % 128 != 0 || K % extra != 0) return 0;
            int sms = 0;
            if (M > kQ4GemvMaxM && q4_tc_fused(M) && current_device(sms) != Q8_OK) return 0;
            return plan_q4(M, N, K, extra, sms).bytes;
        }
    }
    return 0;
}

q8_status q8_quantize_weight_nvfp4(const float* W, int64_t N, int64_t K, uint8_t* q4, uint8_t* sf,
                                   float* gsc, void* stream) {
    if (!W || !q4 || !sf || !gsc) return Q8_ERR_NULL;
    if (N < 1 || N > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (K % 32) return Q8_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(q4) || !aligned16(sf) || !aligned4(gsc)) return Q8_ERR_ALIGN;
    int sms = 0;
    Q8_TRY(current_device(sms));
    return launched(launch_quantize_weight_nvfp4(W, N, (int)K, q4, sf, gsc, (cudaStream_t)stream,
                                                 sms));
}

q8_status q8_linear_w4a16_nvfp4(const void* x, const uint8_t* q4, const uint8_t* sf,
                                const float* gsc, void* y, q8_dtype yt, int64_t M, int64_t N,
                                int64_t K, void* stream) {
    if (yt != Q8_F32 && yt != Q8_BF16) return Q8_ERR_ARG;
    if (M < 0 || M > 0x7fffffff || N < 1 || N > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (K % 32) return Q8_ERR_SHAPE;
    if (M == 0) return Q8_OK;
    if (!x || !q4 || !sf || !gsc || !y) return Q8_ERR_NULL;
    if (!aligned16(x) || !aligned16(q4) || !aligned16(sf) || !aligned4(gsc)) return Q8_ERR_ALIGN;
    int sms = 0;
    Q8_TRY(current_device(sms));
    return launched(launch_w4a16_nvfp4((const uint16_t*)x, q4, sf, gsc, y, yt == Q8_BF16, M, N,
                                       (int)K, (cudaStream_t)stream));
}

q8_status q8_hessian_accumulate(const float* x, int64_t R, int64_t K, double* H, int reset,
                                void* stream) {
    if (R < 0 || R > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (R == 0 && !reset) return Q8_OK;
    if (!H || (R > 0 && !x)) return Q8_ERR_NULL;
    if ((x && !aligned16(x)) || !aligned16(H)) return Q8_ERR_ALIGN;
    int sms = 0;
    Q8_TRY(current_device(sms));
    return launched(launch_hessian_accumulate(x, R, (int)K, H, reset, (cudaStream_t)stream));
}

q8_status q8_gptq_int8(const float* W, const double* H, int64_t N, int64_t K, double damp,
                       int64_t block, int8_t* q, float* s_w, int32_t* wsum, void* workspace,
                       size_t ws_bytes, void* stream) {
    if (N < 1 || N > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (K > kGptqMaxK) return Q8_ERR_SHAPE;
    if (!gptq_block_ok(block) || !isfinite(damp) || damp < 0.0) return Q8_ERR_ARG;
    if (!W || !H || !q || !s_w) return Q8_ERR_NULL;
    if (!aligned16(W) || !aligned16(H) || !aligned16(q) || !aligned4(wsum)) return Q8_ERR_ALIGN;
    const GptqPlan plan = plan_gptq(N, K);
    if (!workspace || ws_bytes < plan.bytes) return Q8_ERR_WORKSPACE;
    if (!aligned16(workspace)) return Q8_ERR_ALIGN;
    int sms = 0;
    int* status = nullptr;
    Q8_TRY(current_device(sms, &status));
    return launched(launch_gptq_int8(W, H, N, (int)K, damp, (int)block, q, s_w, wsum, workspace,
                                     (cudaStream_t)stream, sms, status));
}

q8_status q8_linear_w8a8(const float* x, q8_qparams first, const q8_qparams* second,
                         const int8_t* q, const int32_t* wsum, const float* s_w, float* y,
                         int64_t M, int64_t N, int64_t K, void* workspace, size_t ws_bytes,
                         void* stream) {
    return q8_linear_w8a8_bias(x, first, second, q, wsum, s_w, nullptr, y, M, N, K, workspace,
                               ws_bytes, stream);
}

q8_status q8_linear_w8a8_bias(const float* x, q8_qparams first, const q8_qparams* second,
                              const int8_t* q, const int32_t* wsum, const float* s_w,
                              const float* bias, float* y, int64_t M, int64_t N, int64_t K,
                              void* workspace, size_t ws_bytes, void* stream) {
    Q8_TRY(w8a8_check_args(x, first, second, q, wsum, s_w, bias, y, M, N, K));
    if (M == 0) return Q8_OK;
    const int two = second != nullptr;
    const W8A8Plan plan = plan_w8a8(M, N, K, two);
    if (plan.bytes > 0 && (!workspace || ws_bytes < plan.bytes)) return Q8_ERR_WORKSPACE;
    if (!aligned16(workspace)) return Q8_ERR_ALIGN;
    int sms = 0;
    int* status = nullptr;
    Q8_TRY(current_device(sms, &status));
    cudaStream_t st = (cudaStream_t)stream;
    const float s2 = two ? second->scale : 1.0f;
    const int z2 = two ? second->zero_point : 0;
    if (w8a8_uses_gemv(M, N, K, two))
        return launched(launch_w8a8_gemv(x, first.scale, first.zero_point, two, s2, z2, q, wsum,
                                         s_w, bias, y, M, N, (int)K, st));
    int8_t* xq1 = (int8_t*)workspace + plan.xq1;
    int8_t* xq2 = two ? (int8_t*)workspace + plan.xq2 : nullptr;
    Q8_TRY(launched(launch_quantize_static(x, M, (int)K, first.scale, first.zero_point, two, s2,
                                           z2, xq1, xq2, st, sms)));
    return launched(launch_w8a8_tc(xq1, xq2, first.scale, first.zero_point, two, s2, z2, q, wsum,
                                   s_w, bias, y, M, N, (int)K, st, sms, status));
}

q8_status q8_linear_dq8ca_q4gsw(const void* x, const uint8_t* q4, const float* gs, int G,
                                float* y, int64_t M, int64_t N, int64_t K, void* workspace,
                                size_t ws_bytes, void* stream) {
    if (!valid_group(G)) return Q8_ERR_ARG;
    if (M < 0 || M > 0x7fffffff || N < 1 || N > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (K % 128 != 0 || K % G != 0) return Q8_ERR_SHAPE;
    if (M == 0) return Q8_OK;
    if (!x || !q4 || !gs || !y) return Q8_ERR_NULL;
    if (!aligned16(x) || !aligned16(q4) || !aligned16(gs) || !aligned16(y)) return Q8_ERR_ALIGN;
    int sms = 0;
    int* status = nullptr;
    Q8_TRY(current_device(sms, &status));
    const Q4Plan plan = plan_q4(M, N, K, G, sms);
    if (!workspace || ws_bytes < plan.bytes) return Q8_ERR_WORKSPACE;
    if (!aligned16(workspace)) return Q8_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t* ws = (uint8_t*)workspace;
    float* s = (float*)(ws + plan.s);
    int32_t* z = (int32_t*)(ws + plan.z);
    if (plan.tc) {
        uint16_t* xz = (uint16_t*)(ws + plan.xq);
        if (q4_tc_fused(M)) {
            void* fws = ws + plan.wb;
            Q8_TRY(launched(launch_choose_qparams_shifted((const uint16_t*)x, M, (int)K, s, z, xz, st)));
            return launched(launch_q4_gemm_fused(q4, xz, gs, s, y, G, M, N, (int)K, fws, st, sms,
                                                 status));
        }
        if (plan.i8) {
            int8_t* xq8 = (int8_t*)(ws + plan.xq);
            float* sums16 = (float*)(ws + plan.wb);
            Q8_TRY(launched(launch_choose_qparams((const uint16_t*)x, M, (int)K, s, z, xq8, st)));
            Q8_TRY(launched(launch_q4_group_sums16(q4, N, (int)K, G, sums16, st, sms)));
            return launched(launch_q4_gemm_i8(xq8, z, s, q4, gs, sums16, y, G, M, N, (int)K, st,
                                              sms, status));
        }
        uint16_t* wb = (uint16_t*)(ws + plan.wb);
        Q8_TRY(launched(launch_q4_expand_bf16(q4, N, (int)K, wb, st, sms)));
        Q8_TRY(launched(launch_choose_qparams_shifted((const uint16_t*)x, M, (int)K, s, z, xz, st)));
        return launched(launch_q4_gemm_tc(wb, xz, gs, s, y, G, M, N, (int)K, st, sms, status));
    }
    int8_t* xq = (int8_t*)(ws + plan.xq);
    const bool tma = q4_tma_fits(M, K, G);
    const bool qp = tma && q4_tma_quantizes(M);      // one kernel: qparams + weight stream
    if (!qp) Q8_TRY(launched(launch_choose_qparams((const uint16_t*)x, M, (int)K, s, z, xq, st)));
    if (tma)
        return launched(launch_q4_tma((const uint16_t*)x, xq, s, z, qp, q4, gs, G, y, M, N,
                                      (int)K, st, sms, status));
    return launched(launch_q4_gemv(xq, s, z, q4, gs, G, y, M, N, (int)K, st));
}

q8_status q8_gemm_s8s8_s32(const int8_t* a, const int8_t* b, int32_t* acc, int64_t M, int64_t N,
                           int64_t K, void* stream) {
    if (M < 0 || M > 0x7fffffff || N < 1 || N > 0x7fffffff) return Q8_ERR_SHAPE;
    Q8_TRY(check_k(K));
    if (K < kTcMinK) return Q8_ERR_SHAPE;
    if (M == 0) return Q8_OK;
    if (!a || !b || !acc) return Q8_ERR_NULL;
    if (!aligned16(a) || !aligned16(b) || !aligned16(acc)) return Q8_ERR_ALIGN;
    int sms = 0;
    int* status = nullptr;
    Q8_TRY(current_device(sms, &status));
    return launched(launch_gemm_s8s8_s32_tc(a, b, acc, M, N, (int)K, (cudaStream_t)stream, sms,
                                           status));
}

q8_status q8_selftest_bounded_wait(int64_t limit_ns, int32_t* result, void* stream) {
    if (!result) return Q8_ERR_NULL;
    if (limit_ns < 1000 || limit_ns > 2000000000LL) return Q8_ERR_ARG;
    int sms = 0;
    int* status = nullptr;
    Q8_TRY(current_device(sms, &status));
    k_selftest_bounded_wait<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)limit_ns,
                                                                 status, result);
    return launched(cudaGetLastError());
}

q8_status q8_last_device_status(void* stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return Q8_ERR_LAUNCH;
    }
    return read_and_clear_device_status();
}

}  // extern "C"
