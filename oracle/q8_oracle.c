/*
 * q8_oracle.c -- plain, slow CPU oracle for the int8 quantized linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library; it is written from the
 * definitions on the source pages:
 *
 *   [SmolVLM-Q8]  export/_smolvlm_q8.py (SmolVLM-500M-Instruct ExecuTorch WebGPU recipe)
 *   [ROCm-INT8]   code/quant/int8_linear.py (Ming-Image-0.1-Design ROCm INT8)
 *   [tiny-llm]    src/tinyllm/quant.py (tiny-llm, "INT8 weight-only quantization")
 *   [ET-21229]    pytorch/executorch PR #21229, "Add linear_dq8ca_q4gsw +
 *                 choose_qparams_affine (8da4w)"
 *
 * Conventions
 *   - fp32 steps that decide an integer code are done in fp32 exactly as the
 *     pages' torch code does them: one IEEE operation at a time, no fused
 *     multiply-add (build with -ffp-contract=off, no fast-math), rounding with
 *     nearbyintf() in the default round-to-nearest-even mode (torch.round).
 *   - dot products are accumulated sequentially in k, in fp64 (float inputs)
 *     or int64 (integer inputs); results are returned in fp64 so that the
 *     caller can round them once to the output type.
 *   - parallelism (OpenMP) is over output rows only; every sum runs in one
 *     thread in a fixed order, so results do not depend on the thread count.
 *
 * Parity pins: every function here is checked by the CPU test suite against
 * hand-worked values, closed forms and brute force (see tests/test_oracle_*.py).
 */
#include <math.h>
#include <float.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#include "q8_oracle.h"

/* ------------------------------------------------------------------ helpers */

/* bf16 bits -> fp32 value (exact: bf16 is the top half of an fp32). */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static float clampf(float v, float lo, float hi) {
    if (v < lo) return lo;
    if (v > hi) return hi;
    return v;
}

int q8o_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void q8o_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* --------------------------------------------------- weight quantization (a1)
 * [ROCm-INT8] quantize_weight and QUANT_RULE: per output channel (row n),
 * scale = absmax(row) / 127 in fp32; q = clamp(round(w / scale), -127, 127);
 * a row whose scale comes out 0 gets scale 1.0 and all codes 0.
 * [tiny-llm] module docstring: same grid (s_j = max|W_j| / 127, clip to +-127).
 * wsum[n] = sum_k q[n,k] is the per-row code sum that [SmolVLM-Q8]'s delegated
 * op linear_q8ta_q8csw takes as its weight_sums operand (fix_q8ta_fake).
 * Returns 0, or 1 if a code sum does not fit int32.
 */
int q8o_quantize_weight(const float* W, int64_t N, int64_t K,
                        int8_t* q, float* s, int32_t* wsum) {
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t n = 0; n < N; ++n) {
        const float* w = W + n * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(w[k]);
            if (a > amax) amax = a;
        }
        float scale = amax / 127.0f;          /* fp32 IEEE division */
        int zero = (scale == 0.0f);
        if (zero) scale = 1.0f;
        int64_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            int code = 0;
            if (!zero) {
                float r = nearbyintf(w[k] / scale);   /* true division, ties to even */
                r = clampf(r, -127.0f, 127.0f);
                code = (int)r;
            }
            q[n * K + k] = (int8_t)code;
            sum += code;
        }
        s[n] = scale;
        if (wsum) {
            if (sum > INT32_MAX || sum < INT32_MIN) bad = 1;
            wsum[n] = (int32_t)sum;
        }
    }
    return bad;
}

/* ------------------------------------- weight quantization, observer grid (f1)
 * [SmolVLM-Q8] weight_int8: the codes span the full int8 range [-128, 127] and the
 * per-channel scale comes from torchao's per-channel symmetric min/max observer, whose
 * rule the page states as amax / 127.5.  Written out per row n (the observer's steps,
 * the pages' order; fp32 throughout):
 *   lo = min(min_k w, 0), hi = max(max_k w, 0)         (range widened to contain 0)
 *   amax = max(-lo, hi)
 *   scale = amax / ((127 - (-128)) / 2) = amax / 127.5  (fp32 IEEE division)
 *   scale = max(scale, FLT_EPSILON)                     (the observer's eps floor)
 *   q = clamp(round(w / scale), -128, 127)              (true division, ties to even)
 * An all-zero row therefore gets scale FLT_EPSILON and all codes 0.
 * Returns 0, or 1 if a code sum does not fit int32.
 */
int q8o_quantize_weight_full128(const float* W, int64_t N, int64_t K,
                                int8_t* q, float* s, int32_t* wsum) {
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t n = 0; n < N; ++n) {
        const float* w = W + n * K;
        float lo = 0.0f, hi = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (w[k] < lo) lo = w[k];
            if (w[k] > hi) hi = w[k];
        }
        const float amax = (-lo > hi) ? -lo : hi;
        const float half_range = (127.0f - (-128.0f)) / 2.0f;    /* 127.5, exact */
        float scale = amax / half_range;
        if (scale < FLT_EPSILON) scale = FLT_EPSILON;
        int64_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            float r = nearbyintf(w[k] / scale);
            r = clampf(r, -128.0f, 127.0f);
            const int code = (int)r;
            q[n * K + k] = (int8_t)code;
            sum += code;
        }
        s[n] = scale;
        if (wsum) {
            if (sum > INT32_MAX || sum < INT32_MIN) bad = 1;
            wsum[n] = (int32_t)sum;
        }
    }
    return bad;
}

/* ------------------------------------------ affine activation qparams (a2, R5)
 * The pages use torchao's per-tensor MinMaxObserver ([SmolVLM-Q8] act_observer,
 * qparams) and per-row choose_qparams_affine ([ET-21229]) without printing the
 * formula.  This is the textbook asymmetric int8 scheme both implement:
 *   range widened to contain 0:  mn = min(min x, 0), mx = max(max x, 0)
 *   scale      s = (mx - mn) / 255                (fp32), floored at FLT_EPSILON
 *   zero point z = clamp(-128 - round(mn / s), -128, 127)
 * An all-zero range therefore gives s = FLT_EPSILON, z = -128.
 */
void q8o_qparams_from_minmax(float mn, float mx, float* s_out, int32_t* z_out) {
    if (mn > 0.0f) mn = 0.0f;
    if (mx < 0.0f) mx = 0.0f;
    float scale = (mx - mn) / 255.0f;
    if (scale < FLT_EPSILON) scale = FLT_EPSILON;
    float zf = -128.0f - nearbyintf(mn / scale);
    zf = clampf(zf, -128.0f, 127.0f);
    *s_out = scale;
    *z_out = (int32_t)zf;
}

/* One activation code: clamp(round(x * inv) + z, -128, 127), inv = 1/s in fp32.
 * [SmolVLM-Q8] fake_quant and the quantized_decomposed quantize_per_tensor it
 * mirrors multiply by the reciprocal scale rather than dividing. */
static int8_t act_code(float x, float inv, int32_t z) {
    float t = x * inv;
    float r = nearbyintf(t) + (float)z;
    r = clampf(r, -128.0f, 127.0f);
    return (int8_t)(int)r;
}

/* [ET-21229] choose_qparams_affine: per-row asymmetric int8 scale / zero point
 * from the row's min and max, then (optionally) the row's codes with them. */
void q8o_choose_qparams(const uint16_t* x, int64_t M, int64_t K,
                        float* s, int32_t* z, int8_t* xq) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * K;
        float mn = 0.0f, mx = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_f32(row[k]);
            if (v < mn) mn = v;
            if (v > mx) mx = v;
        }
        float sc;
        int32_t zp;
        q8o_qparams_from_minmax(mn, mx, &sc, &zp);
        s[m] = sc;
        z[m] = zp;
        if (xq) {
            float inv = 1.0f / sc;
            for (int64_t k = 0; k < K; ++k)
                xq[m * K + k] = act_code(bf16_to_f32(row[k]), inv, zp);
        }
    }
}

/* Running min/max of a float tensor (the per-tensor observer's statistics). */
void q8o_minmax(const float* x, int64_t n, float* mn, float* mx) {
    float lo = x[0], hi = x[0];
    for (int64_t i = 1; i < n; ++i) {
        if (x[i] < lo) lo = x[i];
        if (x[i] > hi) hi = x[i];
    }
    *mn = lo;
    *mx = hi;
}

/* --------------------------------------------- static activation codes (a3)
 * [SmolVLM-Q8] Q8Linear.forward: first pass xq1 = q(x, s1, z1).  With a second
 * pass (module docstring "Two passes"), the residual of the first pass
 *     r = x - fake_quant(x, s1, z1) = x - (xq1 - z1) * s1
 * (each operation rounded to fp32 on its own) is quantized with (s2, z2). */
static void static_quant_run(const float* x, int64_t n, float s1, int32_t z1,
                             int8_t* xq1, int has2, float s2, int32_t z2, int8_t* xq2) {
    float inv1 = 1.0f / s1;
    float inv2 = has2 ? 1.0f / s2 : 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        int8_t c1 = act_code(x[i], inv1, z1);
        xq1[i] = c1;
        if (has2) {
            float d1 = (float)((int32_t)c1 - z1) * s1;
            float r = x[i] - d1;
            xq2[i] = act_code(r, inv2, z2);
        }
    }
}

void q8o_static_quant(const float* x, int64_t M, int64_t K, float s1, int32_t z1,
                      int8_t* xq1, int has2, float s2, int32_t z2, int8_t* xq2) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        static_quant_run(x + m * K, K, s1, z1, xq1 + m * K, has2, s2, z2,
                         has2 ? xq2 + m * K : NULL);
}

/* ------------------------------------------- residual calibration observer (f2)
 * [SmolVLM-Q8] calibrate: with two passes, a second calibration run feeds each linear's
 * observer with x - fake_quant(x, *first), and the observer keeps the min and max of
 * everything it saw.  fake_quant as the page defines it, in fp32 one step at a time:
 *     fake_quant(x, s, z) = (clamp(round(x * (1/s)) + z, -128, 127) - z) * s
 * with 1/s the fp32 reciprocal (the reading the activation codes above use).
 * Writes the min and max of the n residuals (n >= 1). */
void q8o_residual_minmax(const float* x, int64_t n, float s1, int32_t z1,
                         float* mn, float* mx) {
    const float inv = 1.0f / s1;
    float lo = 0.0f, hi = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float q = clampf(nearbyintf(x[i] * inv) + (float)z1, -128.0f, 127.0f);
        float fq = (q - (float)z1) * s1;
        float r = x[i] - fq;
        if (i == 0 || r < lo) lo = r;
        if (i == 0 || r > hi) hi = r;
    }
    *mn = lo;
    *mx = hi;
}

/* ------------------------------------------------------------ W8A16 (a4)
 * [tiny-llm] module docstring (the factorisation identity) and Int8Linear.forward:
 *     y[m,n] = s_w[n] * sum_k x[m,k] * q[n,k]
 * x is bf16, q int8: each product is exact in fp64 and the k-sequential fp64
 * sum rounds at relative 2^-53 per step; the scale is applied once after it.  absum[m,n] = sum_k |x * q| * |s_w| bounds the rounding of any
 * other summation order.  rows == NULL means every row m. */
void q8o_linear_w8a16(const uint16_t* x, const int8_t* q, const float* s_w,
                      int64_t M, int64_t N, int64_t K,
                      const int64_t* rows, int64_t nrows,
                      double* y, double* absum) {
    int64_t R = rows ? nrows : M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < R; ++i) {
        int64_t m = rows ? rows[i] : i;
        const uint16_t* xr = x + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const int8_t* qr = q + n * K;
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = (double)bf16_to_f32(xr[k]) * (double)qr[k];
                acc += p;
                mag += fabs(p);
            }
            y[i * N + n] = acc * (double)s_w[n];
            if (absum) absum[i * N + n] = mag * fabs((double)s_w[n]);
        }
    }
}

/* ------------------------------------------------------ W8A8 (a5, a6)
 * [SmolVLM-Q8] Q8Linear.forward: y = linear(dq(q(x,s1,z1)), dq_per_channel(W8, s_w))
 * and, with a second pass, + linear(dq(q(r,s2,z2)), W8) (same int8 weight, no
 * bias the second time).  Written out:
 *     y[m,n] = s_w[n] * ( s1 * sum_k (xq1 - z1) q  +  s2 * sum_k (xq2 - z2) q )
 * The two integer sums are exact (int64).  acc1/acc2 (optional) return the raw
 * int32 dot products sum_k xq * q, the values the integer MMA accumulates.
 * absum[m,n] = |s_w| * sum_k (|(xq1-z1) s1| + |(xq2-z2) s2|) |q|. */
void q8o_linear_w8a8(const float* x, float s1, int32_t z1,
                     int has2, float s2, int32_t z2,
                     const int8_t* q, const float* s_w,
                     int64_t M, int64_t N, int64_t K,
                     const int64_t* rows, int64_t nrows,
                     double* y, double* absum, int32_t* acc1, int32_t* acc2) {
    int64_t R = rows ? nrows : M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < R; ++i) {
        int64_t m = rows ? rows[i] : i;
        int8_t* c1 = (int8_t*)malloc((size_t)K);
        int8_t* c2 = (int8_t*)calloc((size_t)K, 1);
        static_quant_run(x + m * K, K, s1, z1, c1, has2, s2, z2, c2);
        for (int64_t n = 0; n < N; ++n) {
            const int8_t* qr = q + n * K;
            int64_t t1 = 0, t2 = 0, a1 = 0, a2 = 0, g1 = 0, g2 = 0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t w = qr[k];
                t1 += ((int64_t)c1[k] - z1) * w;
                a1 += (int64_t)c1[k] * w;
                g1 += llabs(((int64_t)c1[k] - z1) * w);
                if (has2) {
                    t2 += ((int64_t)c2[k] - z2) * w;
                    a2 += (int64_t)c2[k] * w;
                    g2 += llabs(((int64_t)c2[k] - z2) * w);
                }
            }
            double v = (double)s1 * (double)t1;
            double mag = (double)s1 * (double)g1;
            if (has2) {
                v += (double)s2 * (double)t2;
                mag += (double)s2 * (double)g2;
            }
            y[i * N + n] = (double)s_w[n] * v;
            if (absum) absum[i * N + n] = fabs((double)s_w[n]) * mag;
            if (acc1) acc1[i * N + n] = (int32_t)a1;
            if (acc2 && has2) acc2[i * N + n] = (int32_t)a2;
        }
        free(c1);
        free(c2);
    }
}

/* --------------------------------------------------- int4 group weights (a7)
 * [ET-21229] names a 4-bit group-symmetric weight ("q4gsw") but prints neither
 * grid nor packing.  Reading taken (the int8 rule of [ROCm-INT8] restated for
 * 4 bits and per group of G consecutive k):
 *   gs[n,g] = absmax(W[n, gG:(g+1)G]) / 7 (fp32); a group whose scale comes out
 *   0 gets gs = 1 and codes 0; q4 = clamp(round(W / gs), -7, 7).
 * Packing: byte k/2 of row n holds code k in its low nibble when k is even and
 * in its high nibble when k is odd (two's complement nibbles). */
void q8o_quantize_weight_q4gs(const float* W, int64_t N, int64_t K, int G,
                              uint8_t* q4, float* gs) {
    int64_t ng = K / G;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const float* w = W + n * K;
        for (int64_t g = 0; g < ng; ++g) {
            float amax = 0.0f;
            for (int64_t k = g * G; k < (g + 1) * G; ++k) {
                float a = fabsf(w[k]);
                if (a > amax) amax = a;
            }
            float scale = amax / 7.0f;
            int zero = (scale == 0.0f);
            if (zero) scale = 1.0f;
            gs[n * ng + g] = scale;
            for (int64_t k = g * G; k < (g + 1) * G; ++k) {
                int code = 0;
                if (!zero) {
                    float r = nearbyintf(w[k] / scale);
                    code = (int)clampf(r, -7.0f, 7.0f);
                }
                uint8_t nib = (uint8_t)(code & 0xF);
                uint8_t* byte = q4 + n * (K / 2) + k / 2;
                if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | nib);
                else              *byte = (uint8_t)((*byte & 0x0F) | (nib << 4));
            }
        }
    }
}

/* Signed value of code k in a packed row (see q8o_quantize_weight_q4gs). */
static int q4_code(const uint8_t* row, int64_t k) {
    int nib = (k & 1) ? (row[k / 2] >> 4) & 0xF : row[k / 2] & 0xF;
    return nib >= 8 ? nib - 16 : nib;
}

/* [ET-21229] linear_dq8ca_q4gsw:
 *     out[m,n] = s[m] * sum_k (xq[m,k] - z[m]) * dequant(w)[n,k]
 * with dequant(w)[n,k] = gs[n, k/G] * q4[n,k].  Evaluated as
 *     s[m] * sum_g gs[n,g] * ( sum_{k in g} (xq - z) q4 )
 * with the inner sums exact (int64) and the outer sum in fp64.
 * absum[m,n] = |s[m]| * sum_g |gs[n,g]| * sum_{k in g} |(xq - z) q4|. */
void q8o_linear_dq8ca_q4gsw(const int8_t* xq, const float* s, const int32_t* z,
                            const uint8_t* q4, const float* gs, int G,
                            int64_t M, int64_t N, int64_t K,
                            const int64_t* rows, int64_t nrows,
                            double* y, double* absum) {
    int64_t R = rows ? nrows : M;
    int64_t ng = K / G;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < R; ++i) {
        int64_t m = rows ? rows[i] : i;
        const int8_t* xr = xq + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* wr = q4 + n * (K / 2);
            double acc = 0.0, mag = 0.0;
            for (int64_t g = 0; g < ng; ++g) {
                int64_t part = 0, pabs = 0;
                for (int64_t k = g * G; k < (g + 1) * G; ++k) {
                    int64_t p = ((int64_t)xr[k] - z[m]) * q4_code(wr, k);
                    part += p;
                    pabs += llabs(p);
                }
                acc += (double)gs[n * ng + g] * (double)part;
                mag += fabs((double)gs[n * ng + g]) * (double)pabs;
            }
            y[i * N + n] = (double)s[m] * acc;
            if (absum) absum[i * N + n] = fabs((double)s[m]) * mag;
        }
    }
}

/* Zero-point fold of the 8da4w weight.  In [ET-21229]'s
 *     out[m,n] = s[m] * sum_k (xq[m,k] - z[m]) * dequant(w)[n,k]
 * the zero-point part separates as z[m] * c[n] with c[n] = sum_k dequant(w)[n,k], the row
 * sum of the dequantized weight:
 *     c[n] = sum_g gs[n,g] * (sum_{k in g} q4[n,k])
 * Inner sums exact (int64); each product gs * S is exact in fp64 (24 + 12 bits); the outer
 * sum runs over g ascending in fp64, rounded once to fp32 at the end. */
void q8o_q4gs_zero_fold(const uint8_t* q4, const float* gs, int G, int64_t N, int64_t K,
                        float* c) {
    int64_t ng = K / G;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t* wr = q4 + n * (K / 2);
        double acc = 0.0;
        for (int64_t g = 0; g < ng; ++g) {
            int64_t part = 0;
            for (int64_t k = g * G; k < (g + 1) * G; ++k) part += q4_code(wr, k);
            acc += (double)part * (double)gs[n * ng + g];
        }
        c[n] = (float)acc;
    }
}

/* ------------------------------------------------ NVFP4 weight-only twin (f4)
 * flashrt-structures schemes.py, W4A16Decode: the weights are quantized per 16-element block
 * at bind time to NVFP4 -- E2M1 codes packed two per byte plus block scale factors -- and the
 * activations stay bf16.  The page prints neither the grid nor the scale rule; the reading
 * taken is NVIDIA's NVFP4 layout, the format the name refers to:
 *   E2M1 code: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0; magnitudes
 *     {0, 0.5, 1, 1.5, 2, 3, 4, 6} for codes 0..7 (exponent field 0: 0 and the subnormal 0.5).
 *   E4M3 block scale: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0, no
 *     infinity, 0x7F is NaN, largest finite 448, subnormals m/8 * 2^-6.
 *   per-tensor fp32 scale gsc = amax(W) / (6 * 448)  (1.0 when W is all zero);
 *   per block b of 16 consecutive k in a row:
 *     sb = amax_b / 6;  e = rn_e4m3(sb / gsc);  d = e4m3(e) * gsc      (fp32 steps)
 *     code = rn_e2m1(W / d)  (IEEE division; a block with d == 0 gets codes 0)
 *   rn_* round to the nearest representable value, ties to the even code, and saturate at
 *   the largest finite magnitude; a value that rounds to magnitude 0 gets code 0 (+0).
 *   Packing: byte k/2 of row n holds code k in its low nibble (k even) or high nibble (k odd);
 *   block scales are bytes [N, K/16].
 *   Dequantized weight: e2m1(code) * e4m3(e) * gsc; the first product is exact (2 + 4
 *   significant bits), so y = gsc * sum_k x * (e2m1 * e4m3). */
static const float k_e2m1_mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float q8o_e2m1_value(int code) {
    const float m = k_e2m1_mag[code & 7];
    return (code & 8) ? -m : m;
}

float q8o_e4m3_value(int byte) {
    const int e = (byte >> 3) & 15, m = byte & 7;
    float v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexpf((float)m / 8.0f, -6);
    else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return (byte & 0x80) ? -v : v;
}

/* Nearest E2M1 code of a finite v (ties to even code, saturating at 6, +0 for zero). */
int q8o_rn_e2m1(float v) {
    const float a = fabsf(v);
    int best = 0;
    for (int c = 1; c < 8; ++c) {
        const float dc = fabsf(a - k_e2m1_mag[c]), db = fabsf(a - k_e2m1_mag[best]);
        if (dc < db || (dc == db && (c & 1) == 0)) best = c;
    }
    if (a >= 6.0f) best = 7;
    if (best == 0) return 0;
    return (v < 0.0f ? 8 : 0) | best;
}

/* Nearest non-negative finite E4M3 byte of a finite v >= 0 (ties to even mantissa,
 * saturating at 448). */
int q8o_rn_e4m3(float v) {
    int best = 0;
    double bd = fabs((double)v);
    for (int b = 1; b < 127; ++b) {             /* 0x7F is NaN */
        const double d = fabs((double)v - (double)q8o_e4m3_value(b));
        if (d < bd || (d == bd && (b & 1) == 0)) {
            best = b;
            bd = d;
        }
    }
    if ((double)v >= 448.0) best = 0x7E;
    return best;
}

int q8o_quantize_weight_nvfp4(const float* W, int64_t N, int64_t K, uint8_t* q4,
                              uint8_t* sf, float* gsc_out) {
    if (K % 16) return -1;
    float amax = 0.0f;
    for (int64_t i = 0; i < N * K; ++i) {
        const float a = fabsf(W[i]);
        if (a > amax) amax = a;
    }
    float gsc = amax / 2688.0f;                 /* 6 * 448 */
    if (gsc == 0.0f) gsc = 1.0f;
    *gsc_out = gsc;
    const int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* w = W + n * K + b * 16;
            float bmax = 0.0f;
            for (int j = 0; j < 16; ++j) {
                const float a = fabsf(w[j]);
                if (a > bmax) bmax = a;
            }
            const float sb = bmax / 6.0f;
            const int e = q8o_rn_e4m3(sb / gsc);
            const float d = q8o_e4m3_value(e) * gsc;
            sf[n * nb + b] = (uint8_t)e;
            for (int j = 0; j < 16; ++j) {
                const int code = d == 0.0f ? 0 : q8o_rn_e2m1(w[j] / d);
                const int64_t k = b * 16 + j;
                uint8_t* byte = q4 + n * (K / 2) + k / 2;
                if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | code);
                else              *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
            }
        }
    }
    return 0;
}

/* W4A16 NVFP4 linear: y[m,n] = gsc * sum_k x[m,k] * (e2m1(q[n,k]) * e4m3(sf[n,k/16])),
 * fp64 sum over k ascending; absum the same sum of magnitudes. */
void q8o_linear_w4a16_nvfp4(const uint16_t* x, const uint8_t* q4, const uint8_t* sf, float gsc,
                            int64_t M, int64_t N, int64_t K,
                            const int64_t* rows, int64_t nrows, double* y, double* absum) {
    int64_t R = rows ? nrows : M;
    const int64_t nb = K / 16;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < R; ++i) {
        int64_t m = rows ? rows[i] : i;
        const uint16_t* xr = x + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* wr = q4 + n * (K / 2);
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                const int code = (k & 1) ? (wr[k / 2] >> 4) & 0xF : wr[k / 2] & 0xF;
                const double w = (double)q8o_e2m1_value(code) *
                                 (double)q8o_e4m3_value(sf[n * nb + k / 16]);
                const double p = (double)bf16_to_f32(xr[k]) * w;
                acc += p;
                mag += fabs(p);
            }
            y[i * N + n] = acc * (double)gsc;
            if (absum) absum[i * N + n] = mag * fabs((double)gsc);
        }
    }
}

/* ------------------------------------------------ int8 GEMM, int32 out (a8)
 * acc[m,n] = sum_k a[m,k] * b[n,k], exact. */
void q8o_gemm_s8s8_s32(const int8_t* a, const int8_t* b,
                       int64_t M, int64_t N, int64_t K,
                       const int64_t* rows, int64_t nrows, int32_t* acc) {
    int64_t R = rows ? nrows : M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < R; ++i) {
        int64_t m = rows ? rows[i] : i;
        for (int64_t n = 0; n < N; ++n) {
            int64_t t = 0;
            for (int64_t k = 0; k < K; ++k)
                t += (int64_t)a[m * K + k] * (int64_t)b[n * K + k];
            acc[i * N + n] = (int32_t)t;
        }
    }
}

/* -------------------------------------------------- GPTQ on the int8 grid (f3)
 * [SmolVLM-Q8] gptq_int8 (Frantar et al. 2022) and hessians, float64 throughout:
 *   H = sum over calibration batches of x^T x (x the linear's fp32 inputs as float64);
 *   scale s[n] from weight_int8 of the ORIGINAL row (observer grid, amax / 127.5);
 *   dead columns (diag(H) == 0): H[k,k] = 1 and w[:,k] = 0;
 *   H += damp * mean(diag(H)) * I;
 *   hinv = upper Cholesky factor of H^-1, computed as the page does: the lower Cholesky
 *          factor L of H, H^-1 = L^-T L^-1 (cholesky_inverse), then the upper factor U of
 *          that (U^T U = H^-1);
 *   columns in order, in blocks of `block`: q = clamp(round(w / s), -128, 127),
 *          e = (w - q s) / U[i,i], the block's later columns w[:, j] -= e U[i, j], and after
 *          the block every later column w[:, j] -= sum_t e_t U[t, j] (one matrix product).
 * The page leaves the library routines' summation orders open; here every sum runs in
 * ascending index order, one fp64 operation at a time (no fused multiply-add), which is
 * the order the GPU implementation follows too.  Rows of W are independent once U exists.
 */

/* out[r][j] = sum_t x[t][rows[r]] * x[t][j] for t = 0..R-1 (ascending; fp32 products are
 * exact in fp64).  rows == NULL means every row. */
void q8o_gram_rows(const float* x, int64_t R, int64_t K, const int64_t* rows, int64_t nrows,
                   double* out) {
    const int64_t NR = rows ? nrows : K;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < NR; ++r) {
        const int64_t i = rows ? rows[r] : r;
        double* o = out + r * K;
        for (int64_t j = 0; j < K; ++j) o[j] = 0.0;
        for (int64_t t = 0; t < R; ++t) {
            const double xi = (double)x[t * K + i];
            const float* xt = x + t * K;
            for (int64_t j = 0; j < K; ++j) o[j] = o[j] + xi * (double)xt[j];
        }
    }
}

/* Lower Cholesky factor, left-looking, row-major L (zeros above the diagonal).
 * Returns 1 if a pivot is not positive (H not positive definite). */
static int chol_lower(const double* A, int64_t K, double* L) {
    for (int64_t i = 0; i < K * K; ++i) L[i] = 0.0;
    for (int64_t j = 0; j < K; ++j) {
        double d = A[j * K + j];
        for (int64_t k = 0; k < j; ++k) d = d - L[j * K + k] * L[j * K + k];
        if (!(d > 0.0)) return 1;
        d = sqrt(d);
        L[j * K + j] = d;
#pragma omp parallel for schedule(static)
        for (int64_t i = j + 1; i < K; ++i) {
            double t = A[i * K + j];
            for (int64_t k = 0; k < j; ++k) t = t - L[i * K + k] * L[j * K + k];
            L[i * K + j] = t / d;
        }
    }
    return 0;
}

/* U (row-major, upper) with U^T U = (H damped)^-1; `dead` (nullable) receives the dead
 * columns.  Returns 0, or 1 if a Cholesky pivot is not positive. */
int q8o_gptq_hinv(const double* H0, int64_t K, double damp, double* U, unsigned char* dead) {
    double* H = malloc(sizeof(double) * K * K);
    double* L = malloc(sizeof(double) * K * K);
    double* Li = malloc(sizeof(double) * K * K);
    int bad = 0;
    memcpy(H, H0, sizeof(double) * K * K);
    for (int64_t k = 0; k < K; ++k) {
        const int d = H[k * K + k] == 0.0;
        if (dead) dead[k] = (unsigned char)d;
        if (d) H[k * K + k] = 1.0;
    }
    double tr = 0.0;
    for (int64_t k = 0; k < K; ++k) tr = tr + H[k * K + k];
    const double add = damp * (tr / (double)K);
    for (int64_t k = 0; k < K; ++k) H[k * K + k] = H[k * K + k] + add;
    bad = chol_lower(H, K, L);
    if (!bad) {
        /* L^-1, column by column (forward substitution) */
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t j = 0; j < K; ++j) {
            for (int64_t i = 0; i < j; ++i) Li[i * K + j] = 0.0;
            Li[j * K + j] = 1.0 / L[j * K + j];
            for (int64_t i = j + 1; i < K; ++i) {
                double t = 0.0;
                for (int64_t k = j; k < i; ++k) t = t - L[i * K + k] * Li[k * K + j];
                Li[i * K + j] = t / L[i * K + i];
            }
        }
        /* H^-1 = L^-T L^-1: entry (i, j) = sum over k >= max(i, j), ascending */
#pragma omp parallel for schedule(dynamic, 4)
        for (int64_t i = 0; i < K; ++i)
            for (int64_t j = i; j < K; ++j) {
                double t = 0.0;
                for (int64_t k = j; k < K; ++k) t = t + Li[k * K + i] * Li[k * K + j];
                H[i * K + j] = t;
                H[j * K + i] = t;
            }
        /* upper factor of H^-1: the transpose of its lower factor */
        bad = chol_lower(H, K, L);
        if (!bad)
            for (int64_t i = 0; i < K; ++i)
                for (int64_t j = 0; j < K; ++j) U[i * K + j] = L[j * K + i];
    }
    free(H);
    free(L);
    free(Li);
    return bad;
}

/* GPTQ codes of the listed rows of W (rows == NULL: all N), scale s[r] and code sum
 * wsum[r] (nullable) per listed row.  Returns 0, or 1 if H is not positive definite. */
int q8o_gptq_int8(const float* W, const double* H, int64_t N, int64_t K, double damp,
                  int64_t block, const int64_t* rows, int64_t nrows, int8_t* q, float* s,
                  int32_t* wsum) {
    double* U = malloc(sizeof(double) * K * K);
    unsigned char* dead = malloc((size_t)K);
    const int bad = q8o_gptq_hinv(H, K, damp, U, dead);
    const int64_t NR = rows ? nrows : N;
    if (!bad) {
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t r = 0; r < NR; ++r) {
            const int64_t n = rows ? rows[r] : r;
            const float* wrow = W + n * K;
            int8_t* qrow = q + r * K;
            float sc;
            int8_t* tmp = malloc((size_t)K);
            q8o_quantize_weight_full128(wrow, 1, K, tmp, &sc, NULL);  /* scale of the original row */
            free(tmp);
            const double sd = (double)sc;
            double* w = malloc(sizeof(double) * K);
            double* err = malloc(sizeof(double) * block);
            for (int64_t k = 0; k < K; ++k) w[k] = dead[k] ? 0.0 : (double)wrow[k];
            int64_t sum = 0;
            for (int64_t i1 = 0; i1 < K; i1 += block) {
                const int64_t i2 = i1 + block < K ? i1 + block : K;
                for (int64_t i = i1; i < i2; ++i) {
                    const double col = w[i];
                    double qc = nearbyint(col / sd);
                    if (qc < -128.0) qc = -128.0;
                    if (qc > 127.0) qc = 127.0;
                    qrow[i] = (int8_t)(int)qc;
                    sum += (int)qc;
                    const double e = (col - qc * sd) / U[i * K + i];
                    for (int64_t j = i; j < i2; ++j) w[j] = w[j] - e * U[i * K + j];
                    err[i - i1] = e;
                }
                for (int64_t j = i2; j < K; ++j) {
                    double p = 0.0;
                    for (int64_t t = i1; t < i2; ++t) p = p + err[t - i1] * U[t * K + j];
                    w[j] = w[j] - p;
                }
            }
            s[r] = sc;
            if (wsum) wsum[r] = (int32_t)sum;
            free(w);
            free(err);
        }
    }
    free(U);
    free(dead);
    return bad;
}

/* ------------------------------------------------------- output rounding
 * Round an fp64 value once to bf16 (8 significant bits, ties to even), returned
 * as its 16-bit pattern.  Used to form "the fp64 result rounded to bf16".
 * Finite normal-range inputs only (the outputs of the linears above). */
uint16_t q8o_round_bf16(double v) {
    if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
    int e;
    double m = frexp(v, &e);                 /* v = m * 2^e, 0.5 <= |m| < 1 */
    double r = nearbyint(ldexp(m, 8));       /* 8 significant bits, ties even */
    double b = ldexp(r, e - 8);              /* exactly a bf16 value */
    float f = (float)b;                      /* exact */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

void q8o_round_bf16_array(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = q8o_round_bf16(v[i]);
}
