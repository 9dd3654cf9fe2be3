/* A plain C99 caller of include/q8.h: every entry point is called through the header's own
 * types with arguments that fail the host-side checks (or need no device), and the status
 * codes are compared with the documented ones.  Built and run by test_c_abi.py. */
#include <stdio.h>
#include <string.h>

#include "q8.h"

static int fails = 0;

static void expect(const char* what, q8_status got, q8_status want) {
    if (got != want) {
        printf("%s: got %d (%s), want %d\n", what, (int)got, q8_status_string(got), (int)want);
        ++fails;
    }
}

int main(void) {
    q8_qparams qp;
    q8_qparams out;
    int s;
    qp.scale = 0.1f;
    qp.zero_point = 0;
    if (q8_version() <= 0) ++fails;
    for (s = Q8_OK; s <= Q8_ERR_DEVICE; ++s)
        if (q8_status_string((q8_status)s) == NULL || strlen(q8_status_string((q8_status)s)) == 0)
            ++fails;
    expect("quantize_weight", q8_quantize_weight(NULL, 4, 64, NULL, NULL, NULL, NULL),
           Q8_ERR_NULL);
    expect("quantize_weight_grid",
           q8_quantize_weight_grid(NULL, 4, 64, (q8_grid)7, NULL, NULL, NULL, NULL), Q8_ERR_ARG);
    expect("choose_qparams", q8_choose_qparams(NULL, Q8_F32, 4, 64, NULL, NULL, NULL, NULL),
           Q8_ERR_ARG);
    expect("quantize_static", q8_quantize_static(NULL, -1, 64, qp, NULL, NULL, NULL, NULL),
           Q8_ERR_SHAPE);
    expect("observe_minmax", q8_observe_minmax(NULL, -1, NULL, 1, NULL), Q8_ERR_SHAPE);
    expect("observe_residual_minmax", q8_observe_residual_minmax(NULL, -1, qp, NULL, 1, NULL),
           Q8_ERR_SHAPE);
    expect("qparams_from_minmax", q8_qparams_from_minmax(-1.0f, 1.0f, &out), Q8_OK);
    if (!(out.scale > 0.0f) || out.zero_point < -128 || out.zero_point > 127) ++fails;
    expect("quantize_weight_q4gs", q8_quantize_weight_q4gs(NULL, 4, 64, 48, NULL, NULL, NULL, NULL),
           Q8_ERR_NULL);
    expect("linear_w8a16", q8_linear_w8a16(NULL, NULL, NULL, NULL, (q8_dtype)7, 1, 16, 64, NULL),
           Q8_ERR_ARG);
    expect("linear_w8a16_bias",
           q8_linear_w8a16_bias(NULL, NULL, NULL, NULL, NULL, (q8_dtype)7, 1, 16, 64, NULL),
           Q8_ERR_ARG);
    expect("linear_w8a8",
           q8_linear_w8a8(NULL, qp, NULL, NULL, NULL, NULL, NULL, -1, 16, 64, NULL, 0, NULL),
           Q8_ERR_SHAPE);
    expect("linear_w8a8_bias",
           q8_linear_w8a8_bias(NULL, qp, NULL, NULL, NULL, NULL, NULL, NULL, -1, 16, 64, NULL, 0,
                               NULL),
           Q8_ERR_SHAPE);
    expect("linear_w8a8_noalloc",
           q8_linear_w8a8_noalloc(NULL, qp, NULL, NULL, NULL, NULL, NULL, 8192, 16, 4096, NULL),
           Q8_ERR_NULL);
    expect("quantize_weight_nvfp4", q8_quantize_weight_nvfp4(NULL, 4, 64, NULL, NULL, NULL, NULL),
           Q8_ERR_NULL);
    expect("linear_w4a16_nvfp4",
           q8_linear_w4a16_nvfp4(NULL, NULL, NULL, NULL, NULL, Q8_BF16, 1, 16, 48, NULL),
           Q8_ERR_SHAPE);
    expect("linear_dq8ca_q4gsw",
           q8_linear_dq8ca_q4gsw(NULL, NULL, NULL, 48, NULL, 1, 16, 256, NULL, 0, NULL),
           Q8_ERR_ARG);
    if (q8_workspace_bytes(Q8_OP_LINEAR_W8A8, 17, 16384, 4096, 0) < 17 * 4096) ++fails;
    if (q8_workspace_bytes(Q8_OP_LINEAR_W8A8, 4, 16, 64, 0) != 0) ++fails;
    if (q8_workspace_bytes(Q8_OP_GPTQ_INT8, 0, 8, 64, 128) < 3 * 64 * 64 * 8) ++fails;
    expect("gemm_s8s8_s32", q8_gemm_s8s8_s32(NULL, NULL, NULL, 4, 0, 256, NULL), Q8_ERR_SHAPE);
    expect("selftest_bounded_wait", q8_selftest_bounded_wait(100000, NULL, NULL), Q8_ERR_NULL);
    expect("hessian_accumulate", q8_hessian_accumulate(NULL, -1, 64, NULL, 1, NULL),
           Q8_ERR_SHAPE);
    expect("gptq_int8",
           q8_gptq_int8(NULL, NULL, 0, 64, 0.01, 128, NULL, NULL, NULL, NULL, 0, NULL),
           Q8_ERR_SHAPE);
    printf("failures: %d\n", fails);
    return fails == 0 ? 0 : 1;
}
