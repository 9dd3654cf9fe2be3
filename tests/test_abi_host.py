"""Host-side checks of the C ABI that need no GPU: the library loads, exports every entry
point that include/q8.h declares, validates arguments before touching the device, and
fails loudly (never computes on the CPU) when no sm_100 device is present."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import int8_quantized_linear_q8_b200 as q8
import oracle
from int8_quantized_linear_q8_b200 import build as q8build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    q8build.build()
    return q8.lib()


def _declared():
    text = open(os.path.join(ROOT, "include", "q8.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(q8_[a-z0-9_]+)\s*\(", text)))


def test_header_declarations_are_exported(L):
    declared = _declared()
    assert len(declared) >= 14
    for name in declared:
        assert hasattr(L, name), f"{name} declared in include/q8.h but not exported"
    assert sorted(q8.SYMBOLS) == declared


def test_status_strings(L):
    for code in range(9):
        assert L.q8_status_string(code)
    assert L.q8_version() >= 100


def test_qparams_from_minmax_host_matches_oracle(L):
    """The host formula is bit-identical to the oracle's on many ranges."""
    rng = np.random.default_rng(3)
    cases = [(-1.0, 3.0), (1.0, 4.0), (-4.0, -1.0), (0.0, 0.0), (-1e-9, 1e-9), (-3000.0, 4.0)]
    cases += [tuple(sorted(rng.normal(0, 10, 2).astype(np.float32).tolist())) for _ in range(500)]
    for mn, mx in cases:
        assert q8.q8_qparams_from_minmax(mn, mx) == oracle.qparams_from_minmax(mn, mx), (mn, mx)


def test_qparams_from_minmax_rejects(L):
    out = q8.q8_qparams()
    assert L.q8_qparams_from_minmax(1.0, -1.0, ctypes.byref(out)) == q8.Q8_ERR_ARG
    assert L.q8_qparams_from_minmax(float("nan"), 1.0, ctypes.byref(out)) == q8.Q8_ERR_ARG
    assert L.q8_qparams_from_minmax(0.0, 1.0, None) == q8.Q8_ERR_NULL


def test_workspace_sizes(L):
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, 0, 16, 64) == 0
    # up to 16 rows (or K < 128) the GEMV computes its codes in registers: no workspace
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, 16, 16, 4096, 1) == 0
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, 300, 16, 64, 1) == 0
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, 17, 16, 128, 0) == 0       # small: GEMV
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, 17, 16384, 4096, 0) >= 17 * 4096
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, 17, 16384, 4096, 1) >= 2 * 17 * 4096
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, 4, 16, 63) == 0      # invalid K


def _up(n):
    return -(-n // 256) * 256


@pytest.mark.parametrize("M,G,i8", [(65, 256, True), (4096, 256, True), (512, 128, True),
                                    (2047, 128, True), (2048, 128, False), (512, 64, False),
                                    (4096, 32, False)])
def test_dq8ca_workspace_layout_above_64_rows(L, M, G, i8):
    """Above 64 rows the 8da4w linear runs the int8 GEMM for G = 256 and for G = 128 below
    2048 rows (int8 codes [M, K], s, z, then the fp32 group code sums [N, K/G]), else the
    bf16 GEMM (bf16 codes [M, K], s, z, then the bf16 weight copy [N, K]); each part on a
    256-byte boundary.  No device is needed to size it."""
    N, K = 11008, 4096
    head = _up(M * K * (1 if i8 else 2)) + 2 * _up(4 * M)
    tail = _up(N * (K // G) * 4) if i8 else _up(N * K * 2)
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_DQ8CA_Q4GSW, M, N, K, G) == head + tail


def _p(v):
    return ctypes.c_void_p(v)


def test_argument_validation_before_device(L):
    """Errors are reported from the arguments alone (no device needed)."""
    good = _p(0x10000)      # never dereferenced: every call below fails validation first
    odd = _p(0x10001)
    qp = q8.q8_qparams(0.1, 0)
    assert L.q8_quantize_weight(None, 4, 64, good, good, None, None) == q8.Q8_ERR_NULL
    assert L.q8_quantize_weight(good, 4, 60, good, good, None, None) == q8.Q8_ERR_SHAPE
    assert L.q8_quantize_weight(good, 4, 65536 + 16, good, good, None, None) == q8.Q8_ERR_SHAPE
    assert L.q8_quantize_weight(good, 0, 64, good, good, None, None) == q8.Q8_ERR_SHAPE
    assert L.q8_quantize_weight(odd, 4, 64, good, good, None, None) == q8.Q8_ERR_ALIGN
    assert L.q8_choose_qparams(good, q8.Q8_F32, 4, 64, good, good, None, None) == q8.Q8_ERR_ARG
    assert L.q8_choose_qparams(good, q8.Q8_BF16, 0, 64, None, None, None, None) == q8.Q8_OK
    assert L.q8_linear_w8a16(good, good, good, good, 7, 1, 16, 64, None) == q8.Q8_ERR_ARG
    assert L.q8_linear_w8a16(good, good, good, good, q8.Q8_BF16, 1, 16, 40, None) == q8.Q8_ERR_SHAPE
    assert L.q8_linear_w8a16(good, good, good, good, q8.Q8_BF16, 0, 16, 64, None) == q8.Q8_OK
    bad_qp = q8.q8_qparams(0.0, 0)
    assert L.q8_linear_w8a8(good, bad_qp, None, good, good, good, good, 1, 16, 64, good, 1024,
                            None) == q8.Q8_ERR_ARG
    assert L.q8_linear_w8a8(good, q8.q8_qparams(0.1, 200), None, good, good, good, good, 1, 16,
                            64, good, 1024, None) == q8.Q8_ERR_ARG
    assert L.q8_linear_w8a8(good, qp, None, good, good, good, good, 17, 16384, 4096, None, 0,
                            None) == q8.Q8_ERR_WORKSPACE
    assert L.q8_linear_w8a8(good, qp, None, good, good, good, good, 17, 16384, 4096, good, 10,
                            None) == q8.Q8_ERR_WORKSPACE
    assert L.q8_quantize_weight_q4gs(good, 4, 64, 48, good, good, None, None) == q8.Q8_ERR_ARG
    assert L.q8_quantize_weight_q4gs(good, 4, 96, 64, good, good, None, None) == q8.Q8_ERR_SHAPE
    assert L.q8_quantize_weight_q4gs(good, 4, 128, 64, good, good, _p(0x10002), None) == \
        q8.Q8_ERR_ALIGN
    # weight grid option and bias entry points
    assert L.q8_quantize_weight_grid(good, 4, 64, 2, good, good, None, None) == q8.Q8_ERR_ARG
    assert L.q8_quantize_weight_grid(good, 4, 60, q8.Q8_GRID_FULL128, good, good, None,
                                     None) == q8.Q8_ERR_SHAPE
    assert L.q8_quantize_weight_grid(odd, 4, 64, q8.Q8_GRID_FULL128, good, good, None,
                                     None) == q8.Q8_ERR_ALIGN
    odd4 = _p(0x10002)                                   # 2-byte aligned: not a float pointer
    assert L.q8_linear_w8a16_bias(good, good, good, odd4, good, q8.Q8_F32, 1, 16, 64,
                                  None) == q8.Q8_ERR_ALIGN
    assert L.q8_linear_w8a16_bias(good, good, good, good, good, 7, 1, 16, 64,
                                  None) == q8.Q8_ERR_ARG
    assert L.q8_linear_w8a16_bias(good, good, good, good, good, q8.Q8_F32, 0, 16, 64,
                                  None) == q8.Q8_OK
    assert L.q8_linear_w8a8_bias(good, qp, None, good, good, good, odd4, good, 1, 16, 64, good,
                                 1024, None) == q8.Q8_ERR_ALIGN
    assert L.q8_linear_w8a8_bias(good, bad_qp, None, good, good, good, good, good, 1, 16, 64,
                                 good, 1024, None) == q8.Q8_ERR_ARG
    # GPTQ and the calibration Hessian
    assert L.q8_hessian_accumulate(good, -1, 64, good, 1, None) == q8.Q8_ERR_SHAPE
    assert L.q8_hessian_accumulate(good, 4, 60, good, 1, None) == q8.Q8_ERR_SHAPE
    assert L.q8_hessian_accumulate(good, 0, 64, good, 0, None) == q8.Q8_OK
    assert L.q8_hessian_accumulate(odd, 4, 64, good, 1, None) == q8.Q8_ERR_ALIGN
    ws_g = q8.q8_workspace_bytes(q8.Q8_OP_GPTQ_INT8, 0, 8, 64, 128)
    assert ws_g >= 3 * 64 * 64 * 8 + 8 * 64 * 8
    assert q8.q8_workspace_bytes(q8.Q8_OP_GPTQ_INT8, 0, 8, 64, 0) == 0
    assert q8.q8_workspace_bytes(q8.Q8_OP_GPTQ_INT8, 0, 8, 16384 + 16, 128) == 0
    assert L.q8_gptq_int8(good, good, 8, 64, 0.01, 0, good, good, None, good, ws_g,
                          None) == q8.Q8_ERR_ARG
    assert L.q8_gptq_int8(good, good, 8, 64, -1.0, 128, good, good, None, good, ws_g,
                          None) == q8.Q8_ERR_ARG
    assert L.q8_gptq_int8(good, good, 8, 64, float("nan"), 128, good, good, None, good, ws_g,
                          None) == q8.Q8_ERR_ARG
    assert L.q8_gptq_int8(good, good, 8, 16400, 0.01, 128, good, good, None, good, ws_g,
                          None) == q8.Q8_ERR_SHAPE
    assert L.q8_gptq_int8(good, good, 8, 64, 0.01, 128, good, good, None, good, ws_g - 8,
                          None) == q8.Q8_ERR_WORKSPACE
    assert L.q8_gptq_int8(good, None, 8, 64, 0.01, 128, good, good, None, good, ws_g,
                          None) == q8.Q8_ERR_NULL
    # static activation codes, the first-pass observer
    qpp = ctypes.byref(qp)
    bad_qpp = ctypes.byref(bad_qp)
    assert L.q8_quantize_static(good, -1, 64, qp, None, good, None, None) == q8.Q8_ERR_SHAPE
    assert L.q8_quantize_static(good, 4, 60, qp, None, good, None, None) == q8.Q8_ERR_SHAPE
    assert L.q8_quantize_static(good, 4, 64, bad_qp, None, good, None, None) == q8.Q8_ERR_ARG
    assert L.q8_quantize_static(good, 4, 64, qp, bad_qpp, good, good, None) == q8.Q8_ERR_ARG
    assert L.q8_quantize_static(good, 0, 64, qp, None, None, None, None) == q8.Q8_OK
    assert L.q8_quantize_static(good, 4, 64, qp, qpp, good, None, None) == q8.Q8_ERR_NULL
    assert L.q8_quantize_static(odd, 4, 64, qp, None, good, None, None) == q8.Q8_ERR_ALIGN
    assert L.q8_observe_minmax(good, -1, good, 1, None) == q8.Q8_ERR_SHAPE
    assert L.q8_observe_minmax(good, 8, None, 1, None) == q8.Q8_ERR_NULL
    assert L.q8_observe_minmax(None, 8, good, 1, None) == q8.Q8_ERR_NULL
    assert L.q8_observe_minmax(None, 0, good, 0, None) == q8.Q8_OK
    assert L.q8_observe_minmax(odd, 8, good, 1, None) == q8.Q8_ERR_ALIGN
    # 8da4w linear
    assert L.q8_linear_dq8ca_q4gsw(good, good, good, 48, good, 1, 16, 256, good, 1 << 20,
                                   None) == q8.Q8_ERR_ARG
    assert L.q8_linear_dq8ca_q4gsw(good, good, good, 128, good, 1, 0, 256, good, 1 << 20,
                                   None) == q8.Q8_ERR_SHAPE
    assert L.q8_linear_dq8ca_q4gsw(good, good, good, 64, good, 1, 16, 192, good, 1 << 20,
                                   None) == q8.Q8_ERR_SHAPE
    assert L.q8_linear_dq8ca_q4gsw(good, good, good, 256, good, 1, 16, 384, good, 1 << 20,
                                   None) == q8.Q8_ERR_SHAPE
    assert L.q8_linear_dq8ca_q4gsw(good, good, good, 128, good, 0, 16, 256, None, 0,
                                   None) == q8.Q8_OK
    assert L.q8_linear_dq8ca_q4gsw(None, good, good, 128, good, 1, 16, 256, good, 1 << 20,
                                   None) == q8.Q8_ERR_NULL
    assert L.q8_linear_dq8ca_q4gsw(good, good, good, 128, odd, 1, 16, 256, good, 1 << 20,
                                   None) == q8.Q8_ERR_ALIGN
    # int8 GEMM test export
    assert L.q8_gemm_s8s8_s32(good, good, good, 4, 0, 256, None) == q8.Q8_ERR_SHAPE
    assert L.q8_gemm_s8s8_s32(good, good, good, 4, 16, 64, None) == q8.Q8_ERR_SHAPE
    assert L.q8_gemm_s8s8_s32(good, good, good, 0, 16, 256, None) == q8.Q8_OK
    assert L.q8_gemm_s8s8_s32(good, None, good, 4, 16, 256, None) == q8.Q8_ERR_NULL
    assert L.q8_gemm_s8s8_s32(good, good, odd, 4, 16, 256, None) == q8.Q8_ERR_ALIGN
    # the allocation-free W8A8 reports argument mistakes exactly as q8_linear_w8a8 does
    assert L.q8_linear_w8a8_noalloc(None, qp, None, good, good, good, good, 4, 16, 64,
                                    None) == q8.Q8_ERR_NULL
    assert L.q8_linear_w8a8_noalloc(good, qp, None, good, good, good, good, 1 << 33, 16, 64,
                                    None) == q8.Q8_ERR_SHAPE
    assert L.q8_linear_w8a8_noalloc(good, bad_qp, None, good, good, good, good, 4, 16, 64,
                                    None) == q8.Q8_ERR_ARG
    assert L.q8_linear_w8a8_noalloc(odd, qp, None, good, good, good, good, 4, 16, 64,
                                    None) == q8.Q8_ERR_ALIGN
    assert L.q8_linear_w8a8_noalloc(good, qp, None, good, good, good, good, 0, 16, 64,
                                    None) == q8.Q8_OK
    # NVFP4 weight-only twin
    assert L.q8_quantize_weight_nvfp4(None, 4, 64, good, good, good, None) == q8.Q8_ERR_NULL
    assert L.q8_quantize_weight_nvfp4(good, 4, 48, good, good, good, None) == q8.Q8_ERR_SHAPE
    assert L.q8_quantize_weight_nvfp4(odd, 4, 64, good, good, good, None) == q8.Q8_ERR_ALIGN
    assert L.q8_linear_w4a16_nvfp4(good, good, good, good, good, 7, 1, 16, 64, None) == \
        q8.Q8_ERR_ARG
    assert L.q8_linear_w4a16_nvfp4(good, good, good, good, good, q8.Q8_BF16, 1, 16, 48,
                                   None) == q8.Q8_ERR_SHAPE
    assert L.q8_linear_w4a16_nvfp4(good, good, good, good, good, q8.Q8_BF16, 0, 16, 64,
                                   None) == q8.Q8_OK
    assert L.q8_linear_w4a16_nvfp4(good, None, good, good, good, q8.Q8_BF16, 1, 16, 64,
                                   None) == q8.Q8_ERR_NULL
    assert L.q8_linear_w4a16_nvfp4(good, good, odd, good, good, q8.Q8_BF16, 1, 16, 64,
                                   None) == q8.Q8_ERR_ALIGN
    # bounded-wait self-test
    assert L.q8_selftest_bounded_wait(100000, None, None) == q8.Q8_ERR_NULL
    assert L.q8_selftest_bounded_wait(10, good, None) == q8.Q8_ERR_ARG
    assert L.q8_selftest_bounded_wait(3000000000, good, None) == q8.Q8_ERR_ARG
    mmp = _p(0x10000)
    assert L.q8_observe_residual_minmax(good, 64, bad_qp, mmp, 1, None) == q8.Q8_ERR_ARG
    assert L.q8_observe_residual_minmax(good, -1, qp, mmp, 1, None) == q8.Q8_ERR_SHAPE
    assert L.q8_observe_residual_minmax(odd, 64, qp, mmp, 1, None) == q8.Q8_ERR_ALIGN
    assert L.q8_observe_residual_minmax(None, 64, qp, mmp, 1, None) == q8.Q8_ERR_NULL
    assert L.q8_observe_residual_minmax(good, 0, qp, mmp, 0, None) == q8.Q8_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU failure mode")
def test_valid_call_without_gpu_fails_loudly(L):
    good = _p(0x10000)
    st = L.q8_quantize_weight(good, 4, 64, good, good, None, None)
    assert st in (q8.Q8_ERR_LAUNCH, q8.Q8_ERR_UNSUPPORTED_ARCH)
    qp = q8.q8_qparams(0.1, 0)
    st = L.q8_linear_w8a8_noalloc(good, qp, None, good, good, good, good, 4, 16, 64, None)
    assert st in (q8.Q8_ERR_LAUNCH, q8.Q8_ERR_UNSUPPORTED_ARCH)
    with pytest.raises((q8.Q8Error, ValueError, RuntimeError)):
        q8.q8_linear_w8a16(torch.zeros(1, 64, dtype=torch.bfloat16),
                           torch.zeros(16, 64, dtype=torch.int8), torch.ones(16))
