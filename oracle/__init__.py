"""CPU oracle for the int8 quantized linear -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.  The arithmetic lives in ``q8_oracle.c`` (plain C,
fp32 where the pages fix fp32, fp64/int64 sums); this module only marshals
numpy arrays across ctypes.

bf16 tensors travel as ``numpy.uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_f32 = ctypes.c_float
_vp = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the oracle shared library."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.q8o_num_threads.restype = ctypes.c_int
        L.q8o_set_num_threads.argtypes = [ctypes.c_int]
        L.q8o_quantize_weight.restype = ctypes.c_int
        L.q8o_quantize_weight.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
        L.q8o_quantize_weight_full128.restype = ctypes.c_int
        L.q8o_quantize_weight_full128.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
        L.q8o_qparams_from_minmax.argtypes = [_f32, _f32, _vp, _vp]
        L.q8o_minmax.argtypes = [_vp, _i64, _vp, _vp]
        L.q8o_residual_minmax.argtypes = [_vp, _i64, _f32, _i32, _vp, _vp]
        L.q8o_choose_qparams.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
        L.q8o_static_quant.argtypes = [_vp, _i64, _i64, _f32, _i32, _vp, ctypes.c_int,
                                       _f32, _i32, _vp]
        L.q8o_linear_w8a16.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _i64, _vp, _vp]
        L.q8o_linear_w8a8.argtypes = [_vp, _f32, _i32, ctypes.c_int, _f32, _i32, _vp, _vp,
                                      _i64, _i64, _i64, _vp, _i64, _vp, _vp, _vp, _vp]
        L.q8o_quantize_weight_q4gs.argtypes = [_vp, _i64, _i64, ctypes.c_int, _vp, _vp]
        L.q8o_linear_dq8ca_q4gsw.argtypes = [_vp, _vp, _vp, _vp, _vp, ctypes.c_int,
                                             _i64, _i64, _i64, _vp, _i64, _vp, _vp]
        L.q8o_q4gs_zero_fold.argtypes = [_vp, _vp, ctypes.c_int, _i64, _i64, _vp]
        L.q8o_e2m1_value.restype = ctypes.c_float
        L.q8o_e2m1_value.argtypes = [ctypes.c_int]
        L.q8o_e4m3_value.restype = ctypes.c_float
        L.q8o_e4m3_value.argtypes = [ctypes.c_int]
        L.q8o_rn_e2m1.restype = ctypes.c_int
        L.q8o_rn_e2m1.argtypes = [_f32]
        L.q8o_rn_e4m3.restype = ctypes.c_int
        L.q8o_rn_e4m3.argtypes = [_f32]
        L.q8o_quantize_weight_nvfp4.restype = ctypes.c_int
        L.q8o_quantize_weight_nvfp4.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
        L.q8o_linear_w4a16_nvfp4.argtypes = [_vp, _vp, _vp, _f32, _i64, _i64, _i64, _vp, _i64,
                                             _vp, _vp]
        L.q8o_gemm_s8s8_s32.argtypes = [_vp, _vp, _i64, _i64, _i64, _vp, _i64, _vp]
        L.q8o_gram_rows.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp]
        L.q8o_gptq_hinv.restype = ctypes.c_int
        L.q8o_gptq_hinv.argtypes = [_vp, _i64, ctypes.c_double, _vp, _vp]
        L.q8o_gptq_int8.restype = ctypes.c_int
        L.q8o_gptq_int8.argtypes = [_vp, _vp, _i64, _i64, ctypes.c_double, _i64, _vp, _i64,
                                    _vp, _vp, _vp]
        L.q8o_round_bf16.restype = ctypes.c_uint16
        L.q8o_round_bf16.argtypes = [ctypes.c_double]
        L.q8o_round_bf16_array.argtypes = [_vp, _i64, _vp]
        _LIB = L
    return _LIB


class use_library:
    """Context manager: route every call to another build of the oracle source (used by
    the mutation tests, which compile a copy with one planted mistake)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _LIB
        self.saved = _LIB
        _LIB = None
        saved_build = _build.build
        _build.build = lambda force=False: self.path
        try:
            lib()
        finally:
            _build.build = saved_build
        return self

    def __exit__(self, *exc):
        global _LIB
        _LIB = self.saved


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(_vp)


def _rows(rows, M):
    if rows is None:
        return None, M
    r = _c(np.asarray(rows), np.int64)
    if r.size and (r.min() < 0 or r.max() >= M):
        raise ValueError("row index out of range")
    return r, r.size


def num_threads() -> int:
    return lib().q8o_num_threads()


def set_num_threads(n: int) -> None:
    lib().q8o_set_num_threads(int(n))


def quantize_weight(W: np.ndarray, grid: str = "sym127"):
    """Per-row symmetric int8 codes -> (q int8 [N,K], s fp32 [N], wsum int32 [N]).
    grid "sym127": [ROCm-INT8] quantize_weight (amax/127, codes +-127);
    grid "full128": [SmolVLM-Q8] weight_int8 (observer scale amax/127.5, codes -128..127)."""
    if grid not in ("sym127", "full128"):
        raise ValueError("grid must be 'sym127' or 'full128'")
    W = _c(W, np.float32)
    N, K = W.shape
    q = np.empty((N, K), np.int8)
    s = np.empty(N, np.float32)
    ws = np.empty(N, np.int32)
    fn = lib().q8o_quantize_weight if grid == "sym127" else lib().q8o_quantize_weight_full128
    if fn(_p(W), N, K, _p(q), _p(s), _p(ws)) != 0:
        raise OverflowError("a row's code sum does not fit int32")
    return q, s, ws


def qparams_from_minmax(mn: float, mx: float):
    """Per-tensor affine int8 (scale, zero point) from an observed min / max."""
    s = np.empty(1, np.float32)
    z = np.empty(1, np.int32)
    lib().q8o_qparams_from_minmax(float(mn), float(mx), _p(s), _p(z))
    return float(s[0]), int(z[0])


def minmax(x: np.ndarray):
    x = _c(x, np.float32).reshape(-1)
    if x.size == 0:
        raise ValueError("empty tensor")
    lo = np.empty(1, np.float32)
    hi = np.empty(1, np.float32)
    lib().q8o_minmax(_p(x), x.size, _p(lo), _p(hi))
    return float(lo[0]), float(hi[0])


def residual_minmax(x: np.ndarray, first):
    """Min and max of the first-pass rounding errors x - fake_quant(x, s1, z1) (the second
    calibration run's observer input)."""
    x = _c(x, np.float32).reshape(-1)
    if x.size == 0:
        raise ValueError("empty tensor")
    lo = np.empty(1, np.float32)
    hi = np.empty(1, np.float32)
    lib().q8o_residual_minmax(_p(x), x.size, float(first[0]), int(first[1]), _p(lo), _p(hi))
    return float(lo[0]), float(hi[0])


def choose_qparams(x_bf16: np.ndarray, want_codes: bool = True):
    """Per-row asymmetric int8 qparams of a bf16 [M,K] tensor -> (s, z, xq|None)."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    s = np.empty(M, np.float32)
    z = np.empty(M, np.int32)
    xq = np.empty((M, K), np.int8) if want_codes else None
    lib().q8o_choose_qparams(_p(x), M, K, _p(s), _p(z), _p(xq))
    return s, z, xq


def static_quant(x: np.ndarray, first, second=None):
    """Static per-tensor activation codes (first pass, and residual pass if given)."""
    x = _c(x, np.float32)
    M, K = x.shape
    xq1 = np.empty((M, K), np.int8)
    xq2 = np.empty((M, K), np.int8) if second is not None else None
    s2, z2 = second if second is not None else (0.0, 0)
    lib().q8o_static_quant(_p(x), M, K, float(first[0]), int(first[1]), _p(xq1),
                           int(second is not None), float(s2), int(z2), _p(xq2))
    return xq1, xq2


def _add_bias(y, a, bias):
    """[ROCm-INT8] Int8Linear / [SmolVLM-Q8] Q8Linear: F.linear adds bias[n] to every row
    (once: the residual pass of the two-pass form is a bias-free linear)."""
    if bias is None:
        return y, a
    b = _c(bias, np.float32).astype(np.float64)
    if b.shape != (y.shape[1],):
        raise ValueError("bias must be [N]")
    return y + b[None, :], a + np.abs(b)[None, :]


def linear_w8a16(x_bf16, q, s_w, rows=None, bias=None):
    """fp64 y [R,N] and magnitude sums [R,N] for the listed rows (all if None); with a
    bias [N], y + bias."""
    x = _c(x_bf16, np.uint16)
    q = _c(q, np.int8)
    s_w = _c(s_w, np.float32)
    M, K = x.shape
    N = q.shape[0]
    r, R = _rows(rows, M)
    y = np.empty((R, N), np.float64)
    a = np.empty((R, N), np.float64)
    lib().q8o_linear_w8a16(_p(x), _p(q), _p(s_w), M, N, K, _p(r), R, _p(y), _p(a))
    return _add_bias(y, a, bias)


def linear_w8a8(x, first, q, s_w, second=None, rows=None, bias=None):
    """fp64 y, magnitude sums, and raw int32 dot products (acc1, acc2|None); with a bias
    [N], the first pass's output carries it (y + bias)."""
    x = _c(x, np.float32)
    q = _c(q, np.int8)
    s_w = _c(s_w, np.float32)
    M, K = x.shape
    N = q.shape[0]
    r, R = _rows(rows, M)
    y = np.empty((R, N), np.float64)
    a = np.empty((R, N), np.float64)
    acc1 = np.empty((R, N), np.int32)
    acc2 = np.empty((R, N), np.int32) if second is not None else None
    s2, z2 = second if second is not None else (0.0, 0)
    lib().q8o_linear_w8a8(_p(x), float(first[0]), int(first[1]), int(second is not None),
                          float(s2), int(z2), _p(q), _p(s_w), M, N, K, _p(r), R,
                          _p(y), _p(a), _p(acc1), _p(acc2))
    y, a = _add_bias(y, a, bias)
    return y, a, acc1, acc2


def quantize_weight_q4gs(W: np.ndarray, G: int):
    """int4 group-symmetric codes, packed two per byte -> (q4 u8 [N,K/2], gs fp32 [N,K/G])."""
    W = _c(W, np.float32)
    N, K = W.shape
    if K % G or K % 2:
        raise ValueError("K must be a multiple of G and of 2")
    q4 = np.zeros((N, K // 2), np.uint8)
    gs = np.empty((N, K // G), np.float32)
    lib().q8o_quantize_weight_q4gs(_p(W), N, K, int(G), _p(q4), _p(gs))
    return q4, gs


def linear_dq8ca_q4gsw(xq, s, z, q4, gs, G, rows=None):
    """fp64 y [R,N] and magnitude sums for the 8da4w linear."""
    xq = _c(xq, np.int8)
    s = _c(s, np.float32)
    z = _c(z, np.int32)
    q4 = _c(q4, np.uint8)
    gs = _c(gs, np.float32)
    M, K = xq.shape
    N = q4.shape[0]
    r, R = _rows(rows, M)
    y = np.empty((R, N), np.float64)
    a = np.empty((R, N), np.float64)
    lib().q8o_linear_dq8ca_q4gsw(_p(xq), _p(s), _p(z), _p(q4), _p(gs), int(G), M, N, K,
                                 _p(r), R, _p(y), _p(a))
    return y, a


def q4gs_zero_fold(q4, gs, G):
    """Zero-point fold of an 8da4w weight: c [N] fp32, the row sums of the dequantized
    weight (sum_g gs[n,g] * sum_{k in g} q4[n,k], fp64 over g ascending, one fp32 rounding)."""
    q4 = _c(q4, np.uint8)
    gs = _c(gs, np.float32)
    N, K2 = q4.shape
    c = np.empty(N, np.float32)
    lib().q8o_q4gs_zero_fold(_p(q4), _p(gs), int(G), N, 2 * K2, _p(c))
    return c


def e2m1_value(code: int) -> float:
    return float(lib().q8o_e2m1_value(int(code)))


def e4m3_value(byte: int) -> float:
    return float(lib().q8o_e4m3_value(int(byte)))


def rn_e2m1(v: float) -> int:
    return int(lib().q8o_rn_e2m1(float(v)))


def rn_e4m3(v: float) -> int:
    return int(lib().q8o_rn_e4m3(float(v)))


def quantize_weight_nvfp4(W: np.ndarray):
    """NVFP4 weight codes -> (q4 u8 [N,K/2], block scales u8 [N,K/16] (E4M3), gsc fp32)."""
    W = _c(W, np.float32)
    N, K = W.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    q4 = np.zeros((N, K // 2), np.uint8)
    sf = np.zeros((N, K // 16), np.uint8)
    g = np.zeros(1, np.float32)
    lib().q8o_quantize_weight_nvfp4(_p(W), N, K, _p(q4), _p(sf), _p(g))
    return q4, sf, np.float32(g[0])


def linear_w4a16_nvfp4(x_bf16, q4, sf, gsc, rows=None):
    """fp64 y [R,N] and magnitude sums for the NVFP4 weight-only linear."""
    x = _c(x_bf16, np.uint16)
    q4 = _c(q4, np.uint8)
    sf = _c(sf, np.uint8)
    M, K = x.shape
    N = q4.shape[0]
    r, R = _rows(rows, M)
    y = np.empty((R, N), np.float64)
    a = np.empty((R, N), np.float64)
    lib().q8o_linear_w4a16_nvfp4(_p(x), _p(q4), _p(sf), float(gsc), M, N, K, _p(r), R,
                                 _p(y), _p(a))
    return y, a


def gemm_s8s8_s32(a, b, rows=None):
    a = _c(a, np.int8)
    b = _c(b, np.int8)
    M, K = a.shape
    N = b.shape[0]
    r, R = _rows(rows, M)
    acc = np.empty((R, N), np.int32)
    lib().q8o_gemm_s8s8_s32(_p(a), _p(b), M, N, K, _p(r), R, _p(acc))
    return acc


def gram(x: np.ndarray, rows=None):
    """x^T x in fp64 for one calibration batch x [R, K] (fp32): rows `rows` (all if None)."""
    x = _c(x, np.float32)
    R, K = x.shape
    r, NR = _rows(rows, K)
    out = np.empty((NR, K), np.float64)
    lib().q8o_gram_rows(_p(x), R, K, _p(r), NR, _p(out))
    return out


def hessian(batches, rows=None):
    """[SmolVLM-Q8] hessians: the first batch's x^T x, then H = H + x^T x for each next batch
    (in order; fp64)."""
    H = None
    for x in batches:
        g = gram(x, rows)
        H = g if H is None else H + g
    return H


def gptq_hinv(H: np.ndarray, damp: float = 0.01):
    """Upper factor U (U^T U = damped H^-1) and the dead-column mask used by gptq_int8."""
    H = _c(H, np.float64)
    K = H.shape[0]
    U = np.empty((K, K), np.float64)
    dead = np.empty(K, np.uint8)
    if lib().q8o_gptq_hinv(_p(H), K, float(damp), _p(U), _p(dead)) != 0:
        raise np.linalg.LinAlgError("H is not positive definite after damping")
    return U, dead.astype(bool)


def gptq_int8(W: np.ndarray, H: np.ndarray, damp: float = 0.01, block: int = 128, rows=None):
    """[SmolVLM-Q8] gptq_int8 -> (q int8 [R,K], s fp32 [R], wsum int32 [R]) for the listed
    rows of W (all if None)."""
    W = _c(W, np.float32)
    H = _c(H, np.float64)
    N, K = W.shape
    r, R = _rows(rows, N)
    q = np.empty((R, K), np.int8)
    s = np.empty(R, np.float32)
    ws = np.empty(R, np.int32)
    if lib().q8o_gptq_int8(_p(W), _p(H), N, K, float(damp), int(block), _p(r), R, _p(q),
                           _p(s), _p(ws)) != 0:
        raise np.linalg.LinAlgError("H is not positive definite after damping")
    return q, s, ws


def round_bf16(y64: np.ndarray) -> np.ndarray:
    """Round fp64 values once to bf16; returns uint16 bit patterns."""
    flat = _c(np.asarray(y64, np.float64).reshape(-1), np.float64)
    out = np.empty(flat.size, np.uint16)
    lib().q8o_round_bf16_array(_p(flat), flat.size, _p(out))
    return out.reshape(np.shape(y64))


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("annotations", "ctypes",
                                                                   "os", "np", "lib")]
