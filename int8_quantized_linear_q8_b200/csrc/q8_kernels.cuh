// q8_kernels.cuh -- launcher declarations and device code shared between kernel files.
#pragma once

#include "q8_common.cuh"

namespace q8 {

// Sixteen static activation codes (first pass, and the two-pass residual's codes):
//   c1 = clamp(round(v * (1/s1)) + z1, -128, 127)
//   r  = v - (c1 - z1) * s1          (fp32 product, then fp32 difference; no FMA)
//   c2 = clamp(round(r * (1/s2)) + z2, -128, 127)
// packed four codes per word, lowest k in the lowest byte.
__device__ __forceinline__ void static_codes16(const float (&v)[16], float s1, float inv1,
                                               float z1f, int has2, float inv2, float z2f,
                                               uint32_t (&o1)[4], uint32_t (&o2)[4]) {
    int c1[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) c1[j] = act_code(v[j], inv1, z1f);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        o1[j] = pack4_s8(c1[4 * j], c1[4 * j + 1], c1[4 * j + 2], c1[4 * j + 3]);
    if (has2) {
        int c2[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float d1 = __fmul_rn(__fsub_rn((float)c1[j], z1f), s1);
            float r = __fsub_rn(v[j], d1);
            c2[j] = act_code(r, inv2, z2f);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o2[j] = pack4_s8(c2[4 * j], c2[4 * j + 1], c2[4 * j + 2], c2[4 * j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) o2[j] = 0u;
    }
}

// q8_abi.cu: host checks shared with the allocation-free entry point
q8_status w8a8_check_args(const float* x, const q8_qparams& first, const q8_qparams* second,
                          const int8_t* q, const int32_t* wsum, const float* s_w,
                          const float* bias, const float* y, int64_t M, int64_t N, int64_t K);
q8_status check_current_device();

// k_w4a16.cu (NVFP4 weight-only twin)
cudaError_t launch_quantize_weight_nvfp4(const float* W, int64_t N, int K, uint8_t* q4,
                                         uint8_t* sf, float* gsc, cudaStream_t st, int num_sms);
cudaError_t launch_w4a16_nvfp4(const uint16_t* x, const uint8_t* q4, const uint8_t* sf,
                               const float* gsc, void* y, int y_bf16, int64_t M, int64_t N, int K,
                               cudaStream_t st);

// k_quant.cu
// full: 0 = amax/127 on +-127, 1 = max(amax/127.5, FLT_EPSILON) on [-128, 127]
cudaError_t launch_quantize_weight(const float* W, int64_t N, int K, int full, int8_t* q,
                                   float* s_w, int32_t* wsum, cudaStream_t st);
cudaError_t launch_choose_qparams(const uint16_t* x, int64_t M, int K, float* s, int32_t* z,
                                  int8_t* xq, cudaStream_t st);
cudaError_t launch_choose_qparams_shifted(const uint16_t* x, int64_t M, int K, float* s,
                                          int32_t* z, uint16_t* xz, cudaStream_t st);
cudaError_t launch_quantize_static(const float* x, int64_t M, int K, float s1, int z1, int has2,
                                   float s2, int z2, int8_t* xq1, int8_t* xq2, cudaStream_t st,
                                   int num_sms);
// residual != 0: observe x - fake_quant(x, s1, z1) instead of x
cudaError_t launch_observe_minmax(const float* x, int64_t n, float* mm, int reset, int residual,
                                  float s1, int z1, cudaStream_t st, int num_sms);
cudaError_t launch_quantize_weight_q4gs(const float* W, int64_t N, int K, int G, uint8_t* q4,
                                        float* gs, cudaStream_t st);
cudaError_t launch_q4gs_zero_fold(const uint8_t* q4, const float* gs, int G, int64_t N, int K,
                                  float* c, cudaStream_t st);

// k_gemv_tma.cu
bool make_tmap_u8_2d(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                     int box_cols, int box_rows, CUtensorMapSwizzle swz);
bool w8a16_tma_fits(int64_t M, int64_t K, bool bias = false);
// bias (nullable, fp32 [N]) is added after the scale in every linear launcher below
cudaError_t launch_w8a16_tma(const uint16_t* x, const int8_t* q, const float* s_w,
                             const float* bias, void* y, int y_bf16, int64_t M, int64_t N, int K,
                             cudaStream_t st, int num_sms, int* status);

// k_gemm_tc.cu
cudaError_t launch_gemm_s8s8_s32_tc(const int8_t* a, const int8_t* b, int32_t* acc, int64_t M,
                                    int64_t N, int K, cudaStream_t st, int num_sms, int* status);
cudaError_t launch_w8a8_tc(const int8_t* xq1, const int8_t* xq2, float s1, int z1, int has2,
                           float s2, int z2, const int8_t* q, const int32_t* wsum,
                           const float* s_w, const float* bias, float* y, int64_t M, int64_t N,
                           int K, cudaStream_t st, int num_sms, int* status);

// k_q4.cu
cudaError_t launch_q4_gemv(const int8_t* xq, const float* s, const int32_t* z, const uint8_t* q4,
                           const float* gs, int G, float* y, int64_t M, int64_t N, int K,
                           cudaStream_t st);

// k_q4_tma.cu
bool q4_tma_fits(int64_t M, int64_t K, int G);
bool q4_tma_quantizes(int64_t M);
// qp: x bf16 [M, K] is quantized in the kernel and xq / s / z receive the codes and
// qparams; otherwise xq / s / z are the qparams kernel's output and x is unused.
cudaError_t launch_q4_tma(const uint16_t* x, int8_t* xq, float* s, int32_t* z, bool qp,
                          const uint8_t* q4, const float* gs, int G, float* y, int64_t M,
                          int64_t N, int K, cudaStream_t st, int num_sms, int* status);

// k_q4_i8.cu
cudaError_t launch_q4_group_sums16(const uint8_t* q4, int64_t N, int K, int G, float* sums16,
                                   cudaStream_t st, int num_sms);
cudaError_t launch_q4_gemm_i8(const int8_t* xq, const int32_t* z, const float* s,
                              const uint8_t* q4, const float* gs, const float* sums16, float* y,
                              int G, int64_t M, int64_t N, int K, cudaStream_t st, int num_sms,
                              int* status);
// k_q4_tc.cu
cudaError_t launch_q4_expand_bf16(const uint8_t* q4, int64_t N, int K, uint16_t* wb,
                                  cudaStream_t st, int num_sms);
// M <= 64: the GEMM expands the packed int4 weight itself (q4 [N, K/2], no bf16 copy)
bool q4_tc_fused(int64_t M);
// Workspace of the fused GEMM's K-split (the parts' partial sums; 0 without a split).
size_t q4_fused_workspace_bytes(int64_t M, int64_t N, int K, int G, int num_sms);
cudaError_t launch_q4_gemm_fused(const uint8_t* q4, const uint16_t* xz, const float* gs,
                                 const float* s, float* y, int G, int64_t M, int64_t N, int K,
                                 void* ws, cudaStream_t st, int num_sms, int* status);
cudaError_t launch_q4_gemm_tc(const uint16_t* wb, const uint16_t* xz, const float* gs,
                              const float* s, float* y, int G, int64_t M, int64_t N, int K,
                              cudaStream_t st, int num_sms, int* status);

// k_gptq.cu
struct GptqPlan {
    size_t buf0, buf1, buf2, w, err, dead, bytes;     // byte offsets in the workspace
};
GptqPlan plan_gptq(int64_t N, int64_t K);
bool gptq_block_ok(int64_t block);
cudaError_t launch_hessian_accumulate(const float* x, int64_t R, int K, double* H, int reset,
                                      cudaStream_t st);
cudaError_t launch_gptq_int8(const float* W, const double* H, int64_t N, int K, double damp,
                             int block, int8_t* q, float* s_w, int32_t* wsum, void* ws,
                             cudaStream_t st, int num_sms, int* status);

// k_gemv.cu
cudaError_t launch_w8a16_gemv(const uint16_t* x, const int8_t* q, const float* s_w,
                              const float* bias, void* y, int y_bf16, int64_t M, int64_t N, int K,
                              cudaStream_t st, int num_sms);
cudaError_t launch_w8a8_gemv(const float* x, float s1, int z1, int has2, float s2, int z2,
                             const int8_t* q, const int32_t* wsum, const float* s_w,
                             const float* bias, float* y, int64_t M, int64_t N, int K,
                             cudaStream_t st);

}  // namespace q8
