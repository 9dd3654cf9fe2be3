/*
 * q8_oracle.h -- the CPU oracle's own declarations (test infrastructure only).
 * Independent of the CUDA library's public header: the two share nothing.
 * All arrays are host memory, row-major, innermost dimension contiguous.
 * bf16 tensors are passed as their uint16 bit patterns.
 */
#ifndef Q8_ORACLE_H
#define Q8_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int  q8o_num_threads(void);
void q8o_set_num_threads(int n);

int  q8o_quantize_weight(const float* W, int64_t N, int64_t K,
                         int8_t* q, float* s, int32_t* wsum);
int  q8o_quantize_weight_full128(const float* W, int64_t N, int64_t K,
                                 int8_t* q, float* s, int32_t* wsum);
void q8o_qparams_from_minmax(float mn, float mx, float* s, int32_t* z);
void q8o_minmax(const float* x, int64_t n, float* mn, float* mx);
void q8o_residual_minmax(const float* x, int64_t n, float s1, int32_t z1,
                         float* mn, float* mx);
void q8o_choose_qparams(const uint16_t* x, int64_t M, int64_t K,
                        float* s, int32_t* z, int8_t* xq);
void q8o_static_quant(const float* x, int64_t M, int64_t K, float s1, int32_t z1,
                      int8_t* xq1, int has2, float s2, int32_t z2, int8_t* xq2);
void q8o_linear_w8a16(const uint16_t* x, const int8_t* q, const float* s_w,
                      int64_t M, int64_t N, int64_t K,
                      const int64_t* rows, int64_t nrows,
                      double* y, double* absum);
void q8o_linear_w8a8(const float* x, float s1, int32_t z1,
                     int has2, float s2, int32_t z2,
                     const int8_t* q, const float* s_w,
                     int64_t M, int64_t N, int64_t K,
                     const int64_t* rows, int64_t nrows,
                     double* y, double* absum, int32_t* acc1, int32_t* acc2);
void q8o_quantize_weight_q4gs(const float* W, int64_t N, int64_t K, int G,
                              uint8_t* q4, float* gs);
void q8o_linear_dq8ca_q4gsw(const int8_t* xq, const float* s, const int32_t* z,
                            const uint8_t* q4, const float* gs, int G,
                            int64_t M, int64_t N, int64_t K,
                            const int64_t* rows, int64_t nrows,
                            double* y, double* absum);
void q8o_q4gs_zero_fold(const uint8_t* q4, const float* gs, int G, int64_t N, int64_t K,
                        float* c);
float q8o_e2m1_value(int code);
float q8o_e4m3_value(int byte);
int  q8o_rn_e2m1(float v);
int  q8o_rn_e4m3(float v);
int  q8o_quantize_weight_nvfp4(const float* W, int64_t N, int64_t K, uint8_t* q4, uint8_t* sf,
                               float* gsc);
void q8o_linear_w4a16_nvfp4(const uint16_t* x, const uint8_t* q4, const uint8_t* sf, float gsc,
                            int64_t M, int64_t N, int64_t K, const int64_t* rows, int64_t nrows,
                            double* y, double* absum);
void q8o_gemm_s8s8_s32(const int8_t* a, const int8_t* b,
                       int64_t M, int64_t N, int64_t K,
                       const int64_t* rows, int64_t nrows, int32_t* acc);
void q8o_gram_rows(const float* x, int64_t R, int64_t K, const int64_t* rows, int64_t nrows,
                   double* out);
int  q8o_gptq_hinv(const double* H0, int64_t K, double damp, double* U, unsigned char* dead);
int  q8o_gptq_int8(const float* W, const double* H, int64_t N, int64_t K, double damp,
                   int64_t block, const int64_t* rows, int64_t nrows, int8_t* q, float* s,
                   int32_t* wsum);
uint16_t q8o_round_bf16(double v);
void q8o_round_bf16_array(const double* v, int64_t n, uint16_t* out);

#ifdef __cplusplus
}
#endif
#endif
