/*
 * q8.h -- C ABI of the B200 (sm_100a) int8 quantized-linear library, libq8.so.
 *
 * The per-output-channel quantized linear
 *
 *     y[m,n] = s_w[n] * sum_k xhat[m,k] * q[n,k]
 *
 * in its weight-only (W8A16), static int8-activation (W8A8, one or two passes)
 * and dynamic int8-activation x int4-group-weight (8da4w) forms, plus the
 * quantizers that produce its operands.  Sources of each definition:
 *
 *   [ROCm-INT8]  code/quant/int8_linear.py (Ming-Image-0.1-Design ROCm INT8):
 *                quantize_weight, QUANT_RULE, Int8Linear
 *   [tiny-llm]   src/tinyllm/quant.py (tiny-llm): module docstring (the
 *                factorisation identity), Int8Linear.forward
 *   [SmolVLM-Q8] export/_smolvlm_q8.py (SmolVLM-500M-Instruct ExecuTorch WebGPU):
 *                module docstring ("Two passes"), fake_quant, Q8Linear,
 *                act_observer, fix_q8ta_fake (linear_q8ta_q8csw operands)
 *   [ET-21229]   pytorch/executorch PR #21229 description: choose_qparams_affine
 *                and linear_dq8ca_q4gsw (8da4w)
 *   [flashrt]    flashrt_structures/schemes.py (flashrt-structures 0.2.0): W8A16Decode and
 *                its NVFP4 twin W4A16Decode
 *
 * Conventions shared by every call
 *   - Pointers named as device pointers must be device memory of the current
 *     CUDA device, owned by the caller (the library allocates nothing and keeps
 *     no pointer after a call returns).  Host-only calls are marked.
 *   - Tensors are row-major with the innermost dimension contiguous and
 *     start on a 16-byte boundary (Q8_ERR_ALIGN otherwise).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Every device call only enqueues work on it and returns before
 *     the work completes; nothing synchronises, nothing aborts.  Argument
 *     errors are detected on the host before anything is enqueued and leave
 *     all outputs untouched.
 *   - Shapes: 0 <= M; 1 <= N; 16 <= K <= 65535 and K % 16 == 0 (int32
 *     accumulators cannot overflow: 255 * 128 * 65535 < 2^31).  M == 0 is a
 *     valid no-op.
 *   - The device must be sm_100 (B200); other devices return
 *     Q8_ERR_UNSUPPORTED_ARCH.  There is no CPU fallback.
 *   - Calls that overlap on the GPU may share nothing they write.
 *   - Per device, the first call made with that device current records the device's
 *     architecture and SM count and the device addresses of the library's own device
 *     variables (its status word, the built-in scratch of q8_linear_w8a8_noalloc); later
 *     calls reuse them.  After cudaDeviceReset those addresses are stale: do not call the
 *     library again in a process that has reset a device it used.
 */
#ifndef Q8_H
#define Q8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    Q8_OK = 0,
    Q8_ERR_NULL = 1,              /* a required pointer is NULL                        */
    Q8_ERR_SHAPE = 2,             /* a size is out of range (see conventions)          */
    Q8_ERR_ALIGN = 3,             /* a pointer is not 16-byte aligned                  */
    Q8_ERR_ARG = 4,               /* another argument is invalid (dtype, G, scale)     */
    Q8_ERR_UNSUPPORTED_ARCH = 5,  /* the current device is not sm_100                  */
    Q8_ERR_LAUNCH = 6,            /* a CUDA runtime / driver call failed               */
    Q8_ERR_WORKSPACE = 7,         /* workspace NULL or smaller than q8_workspace_bytes */
    Q8_ERR_DEVICE = 8             /* a kernel recorded a device-side failure           */
} q8_status;

/* Names of the same two codes in the boundary table this header implements: an invalid
 * dtype is one case of Q8_ERR_ARG, an expired bounded wait one case of Q8_ERR_DEVICE. */
#define Q8_ERR_DTYPE Q8_ERR_ARG
#define Q8_ERR_DEVICE_TIMEOUT Q8_ERR_DEVICE

typedef enum { Q8_F32 = 0, Q8_BF16 = 1 } q8_dtype;

/* Static per-tensor affine activation parameters: real x ~ (code - zero_point) * scale,
 * codes in [-128, 127].  scale must be finite and > 0; zero_point in [-128, 127]. */
typedef struct {
    float scale;
    int32_t zero_point;
} q8_qparams;

/* Which call a workspace is sized for (q8_workspace_bytes). */
typedef enum {
    Q8_OP_LINEAR_W8A8 = 0,
    Q8_OP_LINEAR_DQ8CA_Q4GSW = 1,
    Q8_OP_GPTQ_INT8 = 3             /* q8_gptq_int8 (M unused, extra = block) */
} q8_op;

/* Host.  Human-readable name of a status code (static string). */
const char* q8_status_string(q8_status s);

/* Host.  Library ABI version (major * 10000 + minor * 100 + patch). */
int q8_version(void);

/* ------------------------------------------------------------------ quantizers */

/* Per-output-channel symmetric int8 weight codes.  [ROCm-INT8] quantize_weight and
 * QUANT_RULE; [tiny-llm] module docstring.  For each row n of W:
 *     s_w[n] = absmax(W[n,:]) / 127            (fp32 IEEE division)
 *     q[n,k] = clamp(round(W[n,k] / s_w[n]), -127, 127)   (division, ties to even)
 * and a row whose scale comes out 0 gets s_w[n] = 1.0 and all codes 0.
 * wsum[n] = sum_k q[n,k] (the weight_sums operand of [SmolVLM-Q8]'s delegated
 * linear_q8ta_q8csw), written when wsum != NULL.
 *   W     device fp32 [N, K]  (read)
 *   q     device int8 [N, K]  (written)
 *   s_w   device fp32 [N]     (written)
 *   wsum  device int32 [N]    (written; nullable)
 * Codes and scales are bit-identical to the CPU reference definition. */
q8_status q8_quantize_weight(const float* W, int64_t N, int64_t K,
                             int8_t* q, float* s_w, int32_t* wsum, void* stream);

/* Weight grids of q8_quantize_weight_grid. */
typedef enum {
    /* [ROCm-INT8] quantize_weight: s = absmax / 127, codes in [-127, 127] (the grid of
     * q8_quantize_weight). */
    Q8_GRID_SYM127 = 0,
    /* [SmolVLM-Q8] weight_int8 (per-channel symmetric min/max observer on [-128, 127]):
     *     s_w[n] = max(absmax(W[n,:]) / 127.5, FLT_EPSILON)    (fp32 IEEE division)
     *     q[n,k] = clamp(round(W[n,k] / s_w[n]), -128, 127)   (division, ties to even)
     * An all-zero row gets s_w[n] = FLT_EPSILON and all codes 0; the largest positive
     * element of a row lands on 127 and the largest negative one on -128 or -127. */
    Q8_GRID_FULL128 = 1
} q8_grid;

/* q8_quantize_weight on a chosen grid; same arguments and outputs otherwise (wsum is the
 * code sum on that grid).  Q8_ERR_ARG for an unknown grid.  Every linear below accepts
 * weights of either grid: codes of -128 are exact in the bf16 and int8 operand paths. */
q8_status q8_quantize_weight_grid(const float* W, int64_t N, int64_t K, q8_grid grid,
                                  int8_t* q, float* s_w, int32_t* wsum, void* stream);

/* Per-row asymmetric int8 activation parameters.  [ET-21229] choose_qparams_affine
 * (formula of the per-tensor observer in [SmolVLM-Q8] act_observer), per row m:
 *     mn = min(0, min_k x), mx = max(0, max_k x)
 *     s[m] = max((mx - mn) / 255, FLT_EPSILON)      (fp32)
 *     z[m] = clamp(-128 - round(mn / s[m]), -128, 127)
 *     xq[m,k] = clamp(round(x[m,k] * (1 / s[m])) + z[m], -128, 127)   (if xq != NULL)
 *   x     device bf16 [M, K] (read; xt must be Q8_BF16)
 *   s     device fp32 [M], z device int32 [M], xq device int8 [M, K] (nullable)
 * Bit-identical to the CPU reference definition. */
q8_status q8_choose_qparams(const void* x, q8_dtype xt, int64_t M, int64_t K,
                            float* s, int32_t* z, int8_t* xq, void* stream);

/* Static per-tensor activation codes ([SmolVLM-Q8] Q8Linear.forward, fake_quant):
 *     xq1 = clamp(round(x * (1/s1)) + z1, -128, 127)
 * and, when second != NULL, the two-pass residual codes
 *     r   = x - (xq1 - z1) * s1      (each step rounded to fp32)
 *     xq2 = clamp(round(r * (1/s2)) + z2, -128, 127).
 *   x device fp32 [M, K]; xq1 device int8 [M, K]; xq2 device int8 [M, K] (required
 *   iff second != NULL).  `first` / `*second` are read on the host.
 * This is the activation step q8_linear_w8a8 runs; exported for parity tests and
 * for callers that keep codes. */
q8_status q8_quantize_static(const float* x, int64_t M, int64_t K, q8_qparams first,
                             const q8_qparams* second, int8_t* xq1, int8_t* xq2,
                             void* stream);

/* Per-tensor observer statistics ([SmolVLM-Q8] act_observer / MinMaxObserver: min and
 * max of everything observed).  minmax is a device fp32 [2] = {min, max}; with
 * reset != 0 it is first set to {+inf, -inf}; then it is lowered / raised by the
 * n values of x (device fp32).  n == 0 with reset == 0 is a no-op. */
q8_status q8_observe_minmax(const float* x, int64_t n, float* minmax, int reset,
                            void* stream);

/* Residual observer of the two-pass calibration ([SmolVLM-Q8] calibrate: the second
 * calibration run observes each linear's first-pass rounding error, x - fake_quant(x, first)).
 * Same as q8_observe_minmax on the values
 *     r = x - (xq1 - z1) * s1,   xq1 = clamp(round(x * (1/s1)) + z1, -128, 127)
 * computed with exactly the fp32 steps of q8_quantize_static (so the statistics describe
 * the residual the second pass will quantize).  q8_qparams_from_minmax on the result gives
 * the second pass's (s2, z2).  `first` must satisfy the q8_qparams rules (Q8_ERR_ARG). */
q8_status q8_observe_residual_minmax(const float* x, int64_t n, q8_qparams first, float* minmax,
                                     int reset, void* stream);

/* Host.  Per-tensor affine qparams from an observed range (same formula as
 * q8_choose_qparams): out->scale = max((max(mx,0) - min(mn,0)) / 255, FLT_EPSILON),
 * out->zero_point = clamp(-128 - round(min(mn,0) / scale), -128, 127).
 * Q8_ERR_ARG if mn or mx is not finite or mn > mx. */
q8_status q8_qparams_from_minmax(float mn, float mx, q8_qparams* out);

/* int4 group-symmetric weight codes for the 8da4w linear ([ET-21229] names the
 * "q4gsw" weight; its grid is not printed there, so the int8 rule above is used per
 * group): for each row n and group g of G consecutive k,
 *     gs[n,g] = absmax(W[n, gG:(g+1)G]) / 7        (fp32)
 *     code    = clamp(round(W / gs[n,g]), -7, 7)   (a zero-scale group: gs = 1, codes 0)
 * packed two per byte: byte k/2 of row n holds code k in its low nibble (k even)
 * or its high nibble (k odd).
 * When c != NULL it also receives the zero-point fold of each row: [ET-21229] defines
 * out[m,n] = s[m] * sum_k (xq[m,k] - z[m]) * dequant(w)[n,k], whose zero-point part is
 * z[m] * c[n] with c[n] the row sum of the dequantized weight,
 *     c[n] = sum_g gs[n,g] * sum_{k in g} code[n,k]
 * (exact products, an fp64 sum over g in ascending order, one rounding to fp32), so a
 * caller can apply the zero point once per output instead of per element.
 *   W device fp32 [N, K]; q4 device uint8 [N, K/2]; gs device fp32 [N, K/G];
 *   c device fp32 [N] (nullable; 4-byte aligned).
 *   G in {32, 64, 128, 256} and K % G == 0.
 * Codes, scales and c are bit-identical to the CPU reference definition. */
q8_status q8_quantize_weight_q4gs(const float* W, int64_t N, int64_t K, int G,
                                  uint8_t* q4, float* gs, float* c, void* stream);

/* NVFP4 weight codes for the weight-only twin of the W8A16 decode linear
 * ([flashrt] schemes.py, W4A16Decode: "E2M1 packed + block scale factors", one scale per
 * 16-element block, bf16 activations; the page prints no quantization rule, so NVIDIA's
 * NVFP4 layout is used):
 *     gsc = amax(W) / (6 * 448)              (fp32; 1.0 when W is all zero)
 *     per block b of 16 consecutive k of a row:
 *       sb = amax_b / 6;  e = rn_e4m3(sb / gsc);  d = e4m3(e) * gsc     (fp32 steps)
 *       code = rn_e2m1(W / d)                 (IEEE division; d == 0 gives codes 0)
 * where rn_* round to the nearest representable value with ties to the even code and
 * saturate at the largest finite magnitude (E2M1: sign bit 3, magnitudes 0, .5, 1, 1.5, 2,
 * 3, 4, 6 for codes 0..7; E4M3: exponent bits 6..3 with bias 7, mantissa bits 2..0, largest
 * 448); a value that rounds to magnitude 0 gets code 0.  Byte k/2 of row n holds code k in
 * its low nibble (k even) or high nibble (k odd).
 *   W device fp32 [N, K]; q4 device uint8 [N, K/2]; sf device uint8 [N, K/16] (E4M3 block
 *   scales); gsc device fp32 [1] (written; used as scratch by the call before it is).
 *   K % 32 == 0 (Q8_ERR_SHAPE otherwise).
 * Codes, scale bytes and gsc are bit-identical to the CPU reference definition. */
q8_status q8_quantize_weight_nvfp4(const float* W, int64_t N, int64_t K, uint8_t* q4,
                                   uint8_t* sf, float* gsc, void* stream);

/* -------------------------------------------------------------------- linears */

/* W4A16 with NVFP4 weights, the weight-only twin of q8_linear_w8a16 ([flashrt] schemes.py,
 * W4A16Decode: same decode band, half the weight bytes):
 *     y[m,n] = gsc * sum_k x[m,k] * (e2m1(code[n,k]) * e4m3(sf[n,k/16]))
 * The block-scaled weight e2m1 * e4m3 is exact in bf16 (at most 6 significant bits), so the
 * sum runs on the bf16 tensor cores with fp32 accumulation; gsc and one rounding to yt come
 * last.
 *   x device bf16 [M, K]; q4, sf, gsc as written by q8_quantize_weight_nvfp4 (gsc is read
 *   on the device); y device [M, N] of type yt (Q8_BF16 or Q8_F32).  K % 32 == 0.
 * A GEMV streaming the packed codes from HBM (16 activation rows per pass). */
q8_status q8_linear_w4a16_nvfp4(const void* x, const uint8_t* q4, const uint8_t* sf,
                                const float* gsc, void* y, q8_dtype yt, int64_t M, int64_t N,
                                int64_t K, void* stream);


/* W8A16: bf16 activations times int8 weights, the scale applied after the sum
 * ([tiny-llm] factorisation identity y_j = s_j sum_i x_i q_ji; Int8Linear.forward):
 *     y[m,n] = s_w[n] * sum_k x[m,k] * q[n,k]      (fp32 accumulation, one rounding to yt)
 *   x device bf16 [M, K]; q device int8 [N, K]; s_w device fp32 [N];
 *   y device [M, N] of type yt (Q8_BF16 or Q8_F32).
 * Decode-sized M (1..16) runs as an HBM-streaming GEMV on the tensor cores; larger M
 * is computed in blocks of 16 rows (correct, not tuned for prefill). */
q8_status q8_linear_w8a16(const void* x, const int8_t* q, const float* s_w,
                          void* y, q8_dtype yt, int64_t M, int64_t N, int64_t K,
                          void* stream);

/* q8_linear_w8a16 with a bias ([ROCm-INT8] Int8Linear keeps an optional bias and adds it
 * after the scaled matmul):
 *     y[m,n] = s_w[n] * sum_k x[m,k] * q[n,k] + bias[n]
 * the product and the bias fused in one fp32 multiply-add, then one rounding to yt.
 *   bias device fp32 [N] (4-byte aligned; Q8_ERR_ALIGN otherwise); NULL is q8_linear_w8a16.
 * Same kernels and cost as q8_linear_w8a16 (the bias is read once per output column). */
q8_status q8_linear_w8a16_bias(const void* x, const int8_t* q, const float* s_w,
                               const float* bias, void* y, q8_dtype yt, int64_t M, int64_t N,
                               int64_t K, void* stream);

/* W8A8: static per-tensor int8 activations times per-channel int8 weights
 * ([SmolVLM-Q8] Q8Linear.forward; the delegated op takes weight_sums):
 *     acc1[m,n] = sum_k xq1[m,k] q[n,k]     (int32, exact)
 *     y[m,n]    = s_w[n] * s1 * (acc1 - z1 * wsum[n])
 * and with second != NULL (two-pass residual, same int8 weight, module docstring):
 *     y[m,n]   += s_w[n] * s2 * (acc2 - z2 * wsum[n]),  acc2 = sum_k xq2 q
 * with xq1 / xq2 the codes of q8_quantize_static.  fp32 epilogue.
 *   x device fp32 [M, K]; q device int8 [N, K]; wsum device int32 [N] (as written by
 *   q8_quantize_weight); s_w device fp32 [N]; y device fp32 [M, N].
 *   workspace: device scratch of at least q8_workspace_bytes(Q8_OP_LINEAR_W8A8, M, N,
 *   K, second != NULL) bytes (may be NULL when that is 0); its contents on entry do not
 *   matter and are overwritten.
 * Decode-sized M (<= 16, any M when K < 128, and small problems whose 16-row passes over the
 * weight stay below 6 MB) runs as one GEMV kernel on the warp-level int8 MMA that computes
 * the activation codes in registers (the steps of q8_quantize_static) and needs no
 * workspace.  Larger problems first write the codes to the workspace (q8_quantize_static),
 * then run a tcgen05 int8 GEMM (int32 accumulators in tensor memory) with the zero-point
 * term and both scales in its epilogue. */
q8_status q8_linear_w8a8(const float* x, q8_qparams first, const q8_qparams* second,
                         const int8_t* q, const int32_t* wsum, const float* s_w,
                         float* y, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t ws_bytes, void* stream);

/* q8_linear_w8a8 with a bias.  [SmolVLM-Q8] Q8Linear.forward adds the bias to the first
 * pass only (the residual pass is a bias-free linear), so the bias enters once:
 *     y[m,n] = s_w[n] * (s1 * (acc1 - z1 * wsum[n]) [+ s2 * (acc2 - z2 * wsum[n])]) + bias[n]
 * the last multiply and the bias fused in one fp32 multiply-add.
 *   bias device fp32 [N] (4-byte aligned; Q8_ERR_ALIGN otherwise); NULL is q8_linear_w8a8.
 * Other arguments, workspace and errors as q8_linear_w8a8. */
q8_status q8_linear_w8a8_bias(const float* x, q8_qparams first, const q8_qparams* second,
                              const int8_t* q, const int32_t* wsum, const float* s_w,
                              const float* bias, float* y, int64_t M, int64_t N, int64_t K,
                              void* workspace, size_t ws_bytes, void* stream);

/* 8da4w: dynamic per-row int8 activations folded into the 4-bit group-symmetric
 * weight GEMM ([ET-21229] linear_dq8ca_q4gsw):
 *     (s, z, xq) = q8_choose_qparams(x)
 *     y[m,n] = s[m] * sum_g gs[n,g] * sum_{k in g} (xq[m,k] - z[m]) * q4[n,k]
 * with per-group int32 partial sums and fp32 accumulation across groups.
 *   x device bf16 [M, K]; q4 device uint8 [N, K/2]; gs device fp32 [N, K/G];
 *   y device fp32 [M, N]; G in {32, 64, 128, 256}; K % 128 == 0 and K % G == 0
 *   (Q8_ERR_SHAPE otherwise).
 *   workspace: at least q8_workspace_bytes(Q8_OP_LINEAR_DQ8CA_Q4GSW, M, N, K, G) bytes;
 *   it receives the activation codes, scales and zero points.  Above 64 rows the
 *   contraction runs either as a tcgen05 int8 GEMM (codes expanded to int8 in shared
 *   memory, the zero-point term z[m] * sum_{k in g} q4[n,k] and both scales applied in the
 *   epilogue; used for G = 256, and for G = 128 below 2048 rows) or
 *   as a bf16 GEMM on exact small integers; both give the same fp32 results. */
q8_status q8_linear_dq8ca_q4gsw(const void* x, const uint8_t* q4, const float* gs, int G,
                                float* y, int64_t M, int64_t N, int64_t K,
                                void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------- GPTQ (offline) */

/* Calibration Hessian ([SmolVLM-Q8] hessians): the sum over calibration batches of x^T x,
 * in float64 (the fp32 products are exact; each entry sums its batch's rows in ascending
 * order, then adds to the running total).
 *     H  = x^T x        (reset != 0)        H += x^T x      (reset == 0)
 *   x device fp32 [R, K] (R >= 0); H device fp64 [K, K], symmetric on entry when
 *   reset == 0 (as this call leaves it).  K as the shape conventions; R == 0 with reset
 *   zeroes H. */
q8_status q8_hessian_accumulate(const float* x, int64_t R, int64_t K, double* H, int reset,
                                void* stream);

/* GPTQ on the int8 grid of q8_quantize_weight_grid(Q8_GRID_FULL128) ([SmolVLM-Q8]
 * gptq_int8, Frantar et al. 2022), float64 throughout:
 *   s_w[n] = the observer-grid scale of the ORIGINAL row n of W;
 *   dead columns (H[k,k] == 0): H[k,k] = 1 and W[:,k] = 0;  H += damp * mean(diag H) * I;
 *   U = upper Cholesky factor of H^-1;  columns in order, in blocks of `block`:
 *       q = clamp(round(w / s), -128, 127), e = (w - q s) / U[i,i], the block's later
 *       columns w[:, j] -= e U[i, j]; after the block every later column
 *       w[:, j] -= sum_t e_t U[t, j].
 *   W device fp32 [N, K]; H device fp64 [K, K] (read); q device int8 [N, K]; s_w device
 *   fp32 [N]; wsum device int32 [N] (code sums; nullable).  damp finite, >= 0; block in
 *   [1, 256]; K <= 16384 (the three K x K float64 work matrices); Q8_ERR_ARG / SHAPE.
 *   workspace: q8_workspace_bytes(Q8_OP_GPTQ_INT8, 0, N, K, block) bytes (about
 *   24 K^2 + 2.1 kB N + 8 N K); contents on entry do not matter.
 * Every float64 sum runs in ascending index order, one correctly rounded operation at a
 * time, so the codes are the same bits as that sequential definition.  A Hessian that is
 * not positive definite after damping records a device failure (q8_last_device_status
 * returns Q8_ERR_DEVICE) and leaves q undefined.  Offline: O(K^3 + N K^2) float64 work,
 * thousands of small launches. */
q8_status q8_gptq_int8(const float* W, const double* H, int64_t N, int64_t K, double damp,
                       int64_t block, int8_t* q, float* s_w, int32_t* wsum, void* workspace,
                       size_t ws_bytes, void* stream);

/* Host.  Workspace bytes a linear needs for these sizes (0 if none).  `extra` is
 * "two-pass" (0/1) for Q8_OP_LINEAR_W8A8, G for Q8_OP_LINEAR_DQ8CA_Q4GSW and the block
 * size for Q8_OP_GPTQ_INT8.  The 8da4w size for 17..64 rows also depends on the current
 * device's SM count (it sizes the K split of the 17..64-row GEMM).
 * Returns 0 for invalid arguments as well; the linear then reports the error. */
size_t q8_workspace_bytes(q8_op op, int64_t M, int64_t N, int64_t K, int extra);

/* Integer GEMM with int32 output, acc[m,n] = sum_k a[m,k] * b[n,k] (exact): the
 * tcgen05 int8 MMA path of q8_linear_w8a8 without its epilogue, exported so that the
 * int32 accumulators can be checked bit for bit.
 *   a device int8 [M, K]; b device int8 [N, K]; acc device int32 [M, N]; K >= 128
 *   (Q8_ERR_SHAPE otherwise). */
q8_status q8_gemm_s8s8_s32(const int8_t* a, const int8_t* b, int32_t* acc,
                           int64_t M, int64_t N, int64_t K, void* stream);

/* Allocation-free W8A8.  The source pages have no counterpart to this call: it exists for
 * callers that cannot allocate device memory -- a host runtime that has reserved all
 * device memory for its own pool, a latency-critical loop in which cudaMalloc's implicit
 * device-wide synchronisation is not acceptable, or a plain C caller with no allocator to
 * provide q8_linear_w8a8's workspace.  It computes exactly what q8_linear_w8a8 computes,
 * with the same arguments minus the workspace, using a scratch array built into the
 * library instead:
 *   - limit: the scratch holds Q8_NOALLOC_SCRATCH_BYTES (16 MiB); calls whose
 *     q8_workspace_bytes(Q8_OP_LINEAR_W8A8, M, N, K, second != NULL) exceeds it return
 *     Q8_ERR_WORKSPACE before anything is enqueued;
 *   - every GPU on which the library's device code is loaded holds that 16 MiB until the
 *     process exits;
 *   - the first call on a device (with that device current) looks up the array's device
 *     address once; make that first call before any stream capture;
 *   - all calls share the one array, whose contents carry over from call to call (nothing
 *     in it needs to start at zero: each call overwrites the part it reads).  Calls that
 *     may overlap on the GPU (issued on different streams with no ordering between
 *     them) race on it and give wrong results; order them.  Calls on one stream are
 *     ordered.
 *   - nothing here calls cudaMalloc, cudaFree or any allocating routine. */
#define Q8_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
q8_status q8_linear_w8a8_noalloc(const float* x, q8_qparams first, const q8_qparams* second,
                                 const int8_t* q, const int32_t* wsum, const float* s_w,
                                 float* y, int64_t M, int64_t N, int64_t K, void* stream);

/* Self-test of failure detection: launches one CTA that waits on a barrier nothing will
 * complete, with the given limit (1 us .. 2 s, Q8_ERR_ARG otherwise); the wait gives up,
 * writes 0 to *result (device int32, 1 would mean the barrier completed) and records the
 * expiry in the device status word, which q8_last_device_status then returns as
 * Q8_ERR_DEVICE.  The library's pipelined kernels use the same bounded wait (2 s limit)
 * on every barrier, so a lost arrival ends a kernel with an error instead of a hang. */
q8_status q8_selftest_bounded_wait(int64_t limit_ns, int32_t* result, void* stream);

/* Host, synchronising.  Reads and clears the device status word that kernels with
 * bounded waits set when a wait expires (Q8_OK if none did since the last read).
 * Waits for the given stream first. */
q8_status q8_last_device_status(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* Q8_H */
