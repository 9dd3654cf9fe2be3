"""Python binding of libq8 (include/q8.h): int8 quantized linears on B200 (sm_100a).

This module only marshals arguments: it checks tensor dtypes, shapes and devices,
allocates outputs with torch when the caller does not pass them, and calls the C ABI
through ctypes on torch's current CUDA stream.  Every step of the computation runs in
the library's CUDA kernels; there is no CPU path.  Importing works without a GPU, but
every call fails loudly if the compiled library is missing or no sm_100 device is
current.

Function names are the C ABI's.  Errors raise ``Q8Error`` carrying the q8_status code.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libq8.so")

Q8_OK = 0
Q8_ERR_NULL, Q8_ERR_SHAPE, Q8_ERR_ALIGN, Q8_ERR_ARG = 1, 2, 3, 4
Q8_ERR_UNSUPPORTED_ARCH, Q8_ERR_LAUNCH, Q8_ERR_WORKSPACE, Q8_ERR_DEVICE = 5, 6, 7, 8
Q8_F32, Q8_BF16 = 0, 1
Q8_OP_LINEAR_W8A8, Q8_OP_LINEAR_DQ8CA_Q4GSW = 0, 1
Q8_OP_GPTQ_INT8 = 3
Q8_GRID_SYM127, Q8_GRID_FULL128 = 0, 1
_GRIDS = {"sym127": Q8_GRID_SYM127, "full128": Q8_GRID_FULL128}

# Every entry point of include/q8.h, for export checks.
SYMBOLS = (
    "q8_status_string", "q8_version", "q8_quantize_weight", "q8_choose_qparams",
    "q8_quantize_static", "q8_observe_minmax", "q8_qparams_from_minmax",
    "q8_quantize_weight_q4gs", "q8_linear_w8a16", "q8_linear_w8a8", "q8_linear_dq8ca_q4gsw",
    "q8_workspace_bytes", "q8_gemm_s8s8_s32", "q8_last_device_status",
    "q8_linear_w8a8_noalloc", "q8_selftest_bounded_wait",
    "q8_quantize_weight_grid", "q8_linear_w8a16_bias", "q8_linear_w8a8_bias",
    "q8_observe_residual_minmax", "q8_hessian_accumulate", "q8_gptq_int8",
    "q8_quantize_weight_nvfp4", "q8_linear_w4a16_nvfp4",
)
# Built-in scratch of q8_linear_w8a8_noalloc (bytes).
Q8_NOALLOC_SCRATCH_BYTES = 16 << 20


class Q8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib().q8_status_string(status).decode() if _LIB is not None else str(status)
        super().__init__(f"{where}: {msg} (q8_status {status})")


class q8_qparams(ctypes.Structure):
    _fields_ = [("scale", ctypes.c_float), ("zero_point", ctypes.c_int32)]


_LIB: Optional[ctypes.CDLL] = None
_vp, _i64, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libq8.so is not built ({LIB_PATH}); run "
                          "`python int8_quantized_linear_q8_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    st = ctypes.c_int
    L.q8_status_string.restype = ctypes.c_char_p
    L.q8_status_string.argtypes = [st]
    L.q8_version.restype = ctypes.c_int
    L.q8_quantize_weight.restype = st
    L.q8_quantize_weight.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp, _vp]
    L.q8_quantize_weight_grid.restype = st
    L.q8_quantize_weight_grid.argtypes = [_vp, _i64, _i64, st, _vp, _vp, _vp, _vp]
    L.q8_choose_qparams.restype = st
    L.q8_choose_qparams.argtypes = [_vp, st, _i64, _i64, _vp, _vp, _vp, _vp]
    L.q8_quantize_static.restype = st
    L.q8_quantize_static.argtypes = [_vp, _i64, _i64, q8_qparams, ctypes.POINTER(q8_qparams),
                                     _vp, _vp, _vp]
    L.q8_observe_minmax.restype = st
    L.q8_observe_minmax.argtypes = [_vp, _i64, _vp, st, _vp]
    L.q8_hessian_accumulate.restype = st
    L.q8_hessian_accumulate.argtypes = [_vp, _i64, _i64, _vp, st, _vp]
    L.q8_gptq_int8.restype = st
    L.q8_gptq_int8.argtypes = [_vp, _vp, _i64, _i64, ctypes.c_double, _i64, _vp, _vp, _vp,
                               _vp, _sz, _vp]
    L.q8_observe_residual_minmax.restype = st
    L.q8_observe_residual_minmax.argtypes = [_vp, _i64, q8_qparams, _vp, st, _vp]
    L.q8_qparams_from_minmax.restype = st
    L.q8_qparams_from_minmax.argtypes = [ctypes.c_float, ctypes.c_float,
                                         ctypes.POINTER(q8_qparams)]
    L.q8_quantize_weight_q4gs.restype = st
    L.q8_quantize_weight_q4gs.argtypes = [_vp, _i64, _i64, st, _vp, _vp, _vp, _vp]
    L.q8_quantize_weight_nvfp4.restype = st
    L.q8_quantize_weight_nvfp4.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp, _vp]
    L.q8_linear_w4a16_nvfp4.restype = st
    L.q8_linear_w4a16_nvfp4.argtypes = [_vp, _vp, _vp, _vp, _vp, st, _i64, _i64, _i64, _vp]
    L.q8_linear_w8a16.restype = st
    L.q8_linear_w8a16.argtypes = [_vp, _vp, _vp, _vp, st, _i64, _i64, _i64, _vp]
    L.q8_linear_w8a16_bias.restype = st
    L.q8_linear_w8a16_bias.argtypes = [_vp, _vp, _vp, _vp, _vp, st, _i64, _i64, _i64, _vp]
    L.q8_linear_w8a8.restype = st
    L.q8_linear_w8a8.argtypes = [_vp, q8_qparams, ctypes.POINTER(q8_qparams), _vp, _vp, _vp,
                                 _vp, _i64, _i64, _i64, _vp, _sz, _vp]
    L.q8_linear_w8a8_bias.restype = st
    L.q8_linear_w8a8_bias.argtypes = [_vp, q8_qparams, ctypes.POINTER(q8_qparams), _vp, _vp,
                                      _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz, _vp]
    L.q8_linear_dq8ca_q4gsw.restype = st
    L.q8_linear_dq8ca_q4gsw.argtypes = [_vp, _vp, _vp, st, _vp, _i64, _i64, _i64, _vp, _sz, _vp]
    L.q8_workspace_bytes.restype = _sz
    L.q8_workspace_bytes.argtypes = [st, _i64, _i64, _i64, st]
    L.q8_gemm_s8s8_s32.restype = st
    L.q8_gemm_s8s8_s32.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _vp]
    L.q8_last_device_status.restype = st
    L.q8_last_device_status.argtypes = [_vp]
    L.q8_selftest_bounded_wait.restype = st
    L.q8_selftest_bounded_wait.argtypes = [_i64, _vp, _vp]
    L.q8_linear_w8a8_noalloc.restype = st
    L.q8_linear_w8a8_noalloc.argtypes = [_vp, q8_qparams, ctypes.POINTER(q8_qparams), _vp, _vp,
                                         _vp, _vp, _i64, _i64, _i64, _vp]
    _LIB = L
    return L


def lib() -> ctypes.CDLL:
    """The loaded libq8.so (raises ImportError if it has not been built)."""
    return _lib()


def _check(status: int, where: str) -> None:
    if status != Q8_OK:
        raise Q8Error(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# The current stream's raw handle without building a torch Stream object (that alone took
# ~4.5 us per call, a third of a decode-sized call's host time).
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream=None):
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    if _raw_stream is not None:
        return ctypes.c_void_p(_raw_stream(torch.cuda.current_device()))
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: Tuple[int, ...]):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.shape != shape:
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out(t, name, dtype, shape, device):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    _need(t, name, dtype, shape)
    return t


def _qp(p) -> q8_qparams:
    s, z = p
    return q8_qparams(float(s), int(z))


# ---------------------------------------------------------------------------- quantizers


def q8_quantize_weight(W: torch.Tensor, q=None, s_w=None, wsum=None, want_wsum=True,
                       stream=None, grid: str = "sym127"):
    """Per-row symmetric int8 codes of an fp32 [N, K] weight -> (q, s_w, wsum|None).
    grid "sym127": amax/127 on [-127, 127]; "full128": max(amax/127.5, eps) on [-128, 127]."""
    if grid not in _GRIDS:
        raise ValueError(f"grid must be one of {sorted(_GRIDS)}")
    if W.dim() != 2:
        raise ValueError("W must be 2-D [N, K]")
    N, K = W.shape
    _need(W, "W", torch.float32, (N, K))
    q = _out(q, "q", torch.int8, (N, K), W.device)
    s_w = _out(s_w, "s_w", torch.float32, (N,), W.device)
    if want_wsum or wsum is not None:
        wsum = _out(wsum, "wsum", torch.int32, (N,), W.device)
    _check(_lib().q8_quantize_weight_grid(_ptr(W), N, K, _GRIDS[grid], _ptr(q), _ptr(s_w),
                                          _ptr(wsum), _stream(stream)), "q8_quantize_weight")
    return q, s_w, wsum


def q8_choose_qparams(x: torch.Tensor, s=None, z=None, xq=None, want_codes=True, stream=None):
    """Per-row asymmetric int8 qparams of a bf16 [M, K] tensor -> (s, z, xq|None)."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D [M, K]")
    M, K = x.shape
    _need(x, "x", torch.bfloat16, (M, K))
    s = _out(s, "s", torch.float32, (M,), x.device)
    z = _out(z, "z", torch.int32, (M,), x.device)
    if want_codes or xq is not None:
        xq = _out(xq, "xq", torch.int8, (M, K), x.device)
    _check(_lib().q8_choose_qparams(_ptr(x), Q8_BF16, M, K, _ptr(s), _ptr(z), _ptr(xq),
                                    _stream(stream)), "q8_choose_qparams")
    return s, z, xq


def q8_quantize_static(x: torch.Tensor, first, second=None, xq1=None, xq2=None, stream=None):
    """Static per-tensor codes of an fp32 [M, K] tensor (+ two-pass residual codes)."""
    M, K = x.shape
    _need(x, "x", torch.float32, (M, K))
    xq1 = _out(xq1, "xq1", torch.int8, (M, K), x.device)
    sec = None
    if second is not None:
        xq2 = _out(xq2, "xq2", torch.int8, (M, K), x.device)
        sec = ctypes.byref(_qp(second))
    _check(_lib().q8_quantize_static(_ptr(x), M, K, _qp(first), sec, _ptr(xq1),
                                     _ptr(xq2) if second is not None else None,
                                     _stream(stream)), "q8_quantize_static")
    return xq1, (xq2 if second is not None else None)


def q8_observe_minmax(x: torch.Tensor, minmax: torch.Tensor, reset: bool = False,
                      stream=None) -> torch.Tensor:
    """Lower/raise the device fp32 [2] = {min, max} by the values of x (fp32)."""
    _need(x, "x", torch.float32, tuple(x.shape))
    _need(minmax, "minmax", torch.float32, (2,))
    _check(_lib().q8_observe_minmax(_ptr(x), x.numel(), _ptr(minmax), int(bool(reset)),
                                    _stream(stream)), "q8_observe_minmax")
    return minmax


def q8_observe_residual_minmax(x: torch.Tensor, first, minmax: torch.Tensor,
                               reset: bool = False, stream=None) -> torch.Tensor:
    """Lower/raise {min, max} by the first-pass rounding errors x - fake_quant(x, first)."""
    _need(x, "x", torch.float32, tuple(x.shape))
    _need(minmax, "minmax", torch.float32, (2,))
    _check(_lib().q8_observe_residual_minmax(_ptr(x), x.numel(), _qp(first), _ptr(minmax),
                                             int(bool(reset)), _stream(stream)),
           "q8_observe_residual_minmax")
    return minmax


def q8_qparams_from_minmax(mn: float, mx: float) -> Tuple[float, int]:
    """Host call: per-tensor affine (scale, zero_point) from an observed range."""
    out = q8_qparams()
    _check(_lib().q8_qparams_from_minmax(float(mn), float(mx), ctypes.byref(out)),
           "q8_qparams_from_minmax")
    return float(out.scale), int(out.zero_point)


def q8_quantize_weight_q4gs(W: torch.Tensor, G: int, q4=None, gs=None, stream=None,
                            c=None, want_c: bool = False):
    """int4 group-symmetric codes (packed, low nibble = even k) -> (q4 [N,K/2], gs [N,K/G]);
    with want_c (or a `c` tensor) also the zero-point fold c [N] (row sums of the
    dequantized weight) -> (q4, gs, c)."""
    N, K = W.shape
    _need(W, "W", torch.float32, (N, K))
    if G <= 0 or K % G or K % 2:
        raise ValueError("K must be a multiple of G")
    q4 = _out(q4, "q4", torch.uint8, (N, K // 2), W.device)
    gs = _out(gs, "gs", torch.float32, (N, K // G), W.device)
    fold = want_c or c is not None
    if fold:
        c = _out(c, "c", torch.float32, (N,), W.device)
    _check(_lib().q8_quantize_weight_q4gs(_ptr(W), N, K, int(G), _ptr(q4), _ptr(gs),
                                          _ptr(c) if fold else None, _stream(stream)),
           "q8_quantize_weight_q4gs")
    return (q4, gs, c) if fold else (q4, gs)


def q8_quantize_weight_nvfp4(W: torch.Tensor, q4=None, sf=None, gsc=None, stream=None):
    """NVFP4 weight codes -> (q4 uint8 [N,K/2], sf uint8 [N,K/16] (E4M3 block scales),
    gsc fp32 [1] on the device)."""
    N, K = W.shape
    _need(W, "W", torch.float32, (N, K))
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    q4 = _out(q4, "q4", torch.uint8, (N, K // 2), W.device)
    sf = _out(sf, "sf", torch.uint8, (N, K // 16), W.device)
    gsc = _out(gsc, "gsc", torch.float32, (1,), W.device)
    _check(_lib().q8_quantize_weight_nvfp4(_ptr(W), N, K, _ptr(q4), _ptr(sf), _ptr(gsc),
                                           _stream(stream)), "q8_quantize_weight_nvfp4")
    return q4, sf, gsc


# ---------------------------------------------------------------------------- linears


def q8_linear_w4a16_nvfp4(x: torch.Tensor, q4: torch.Tensor, sf: torch.Tensor,
                          gsc: torch.Tensor, y=None, out_dtype=torch.bfloat16,
                          stream=None) -> torch.Tensor:
    """bf16 activations x NVFP4 weights (codes, E4M3 block scales, device gsc [1])."""
    M, K = x.shape
    N = q4.shape[0]
    _need(x, "x", torch.bfloat16, (M, K))
    _need(q4, "q4", torch.uint8, (N, K // 2))
    _need(sf, "sf", torch.uint8, (N, K // 16))
    _need(gsc, "gsc", torch.float32, (1,))
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    y = _out(y, "y", out_dtype, (M, N), x.device)
    yt = Q8_BF16 if y.dtype == torch.bfloat16 else Q8_F32
    _check(_lib().q8_linear_w4a16_nvfp4(_ptr(x), _ptr(q4), _ptr(sf), _ptr(gsc), _ptr(y), yt,
                                        M, N, K, _stream(stream)), "q8_linear_w4a16_nvfp4")
    return y


def q8_workspace_bytes(op: int, M: int, N: int, K: int, extra: int = 0) -> int:
    return int(_lib().q8_workspace_bytes(int(op), int(M), int(N), int(K), int(extra)))


def _workspace(ws, nbytes, device):
    if nbytes == 0:
        return ws, 0 if ws is None else ws.numel()
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def q8_linear_w8a16(x: torch.Tensor, q: torch.Tensor, s_w: torch.Tensor, y=None,
                    out_dtype: torch.dtype = torch.bfloat16, stream=None,
                    bias: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y[m,n] = s_w[n] * sum_k x[m,k] q[n,k] (+ bias[n]); x bf16 [M,K], q int8 [N,K],
    bias fp32 [N], y bf16|fp32 [M,N]."""
    M, K = x.shape
    N = q.shape[0]
    _need(x, "x", torch.bfloat16, (M, K))
    _need(q, "q", torch.int8, (N, K))
    _need(s_w, "s_w", torch.float32, (N,))
    if bias is not None:
        _need(bias, "bias", torch.float32, (N,))
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    y = _out(y, "y", out_dtype, (M, N), x.device)
    yt = Q8_BF16 if y.dtype == torch.bfloat16 else Q8_F32
    if bias is None:
        _check(_lib().q8_linear_w8a16(_ptr(x), _ptr(q), _ptr(s_w), _ptr(y), yt, M, N, K,
                                      _stream(stream)), "q8_linear_w8a16")
    else:
        _check(_lib().q8_linear_w8a16_bias(_ptr(x), _ptr(q), _ptr(s_w), _ptr(bias), _ptr(y), yt,
                                           M, N, K, _stream(stream)), "q8_linear_w8a16_bias")
    return y


def q8_linear_w8a8(x: torch.Tensor, first, q: torch.Tensor, wsum: torch.Tensor,
                   s_w: torch.Tensor, second=None, y=None, workspace=None,
                   stream=None, bias: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Static int8 activations x int8 weights (one or two passes); fp32 in, fp32 out; an
    fp32 [N] bias is added once (the first pass's)."""
    M, K = x.shape
    N = q.shape[0]
    _need(x, "x", torch.float32, (M, K))
    _need(q, "q", torch.int8, (N, K))
    _need(wsum, "wsum", torch.int32, (N,))
    _need(s_w, "s_w", torch.float32, (N,))
    if bias is not None:
        _need(bias, "bias", torch.float32, (N,))
    y = _out(y, "y", torch.float32, (M, N), x.device)
    nbytes = q8_workspace_bytes(Q8_OP_LINEAR_W8A8, M, N, K, int(second is not None))
    workspace, wsb = _workspace(workspace, nbytes, x.device)
    sec = None if second is None else ctypes.byref(_qp(second))
    if bias is None:
        _check(_lib().q8_linear_w8a8(_ptr(x), _qp(first), sec, _ptr(q), _ptr(wsum), _ptr(s_w),
                                     _ptr(y), M, N, K, _ptr(workspace), wsb, _stream(stream)),
               "q8_linear_w8a8")
    else:
        _check(_lib().q8_linear_w8a8_bias(_ptr(x), _qp(first), sec, _ptr(q), _ptr(wsum),
                                          _ptr(s_w), _ptr(bias), _ptr(y), M, N, K,
                                          _ptr(workspace), wsb, _stream(stream)),
               "q8_linear_w8a8_bias")
    return y


def q8_linear_w8a8_noalloc(x: torch.Tensor, first, q: torch.Tensor, wsum: torch.Tensor,
                           s_w: torch.Tensor, second=None, y=None, stream=None) -> torch.Tensor:
    """q8_linear_w8a8 without a workspace: for callers that cannot allocate device memory.

    The library uses a 16 MiB scratch array of its own (shared by every call on a device;
    calls on different streams must not overlap).  Only `y` is allocated here when the
    caller does not pass it; pass `y` to allocate nothing at all."""
    M, K = x.shape
    N = q.shape[0]
    _need(x, "x", torch.float32, (M, K))
    _need(q, "q", torch.int8, (N, K))
    _need(wsum, "wsum", torch.int32, (N,))
    _need(s_w, "s_w", torch.float32, (N,))
    y = _out(y, "y", torch.float32, (M, N), x.device)
    sec = None if second is None else ctypes.byref(_qp(second))
    _check(_lib().q8_linear_w8a8_noalloc(_ptr(x), _qp(first), sec, _ptr(q), _ptr(wsum),
                                         _ptr(s_w), _ptr(y), M, N, K, _stream(stream)),
           "q8_linear_w8a8_noalloc")
    return y


def q8_hessian_accumulate(x: torch.Tensor, H: Optional[torch.Tensor] = None,
                          reset: bool = False, stream=None) -> torch.Tensor:
    """H (= if reset or H is None, else +=) x^T x in float64; x fp32 [R, K]."""
    R, K = x.shape
    _need(x, "x", torch.float32, (R, K))
    if H is None:
        H = torch.empty(K, K, dtype=torch.float64, device=x.device)
        reset = True
    _need(H, "H", torch.float64, (K, K))
    _check(_lib().q8_hessian_accumulate(_ptr(x), R, K, _ptr(H), int(bool(reset)),
                                        _stream(stream)), "q8_hessian_accumulate")
    return H


def q8_gptq_int8(W: torch.Tensor, H: torch.Tensor, damp: float = 0.01, block: int = 128,
                 q=None, s_w=None, wsum=None, want_wsum=True, workspace=None, stream=None):
    """GPTQ int8 codes of an fp32 [N, K] weight against a float64 [K, K] calibration Hessian
    -> (q int8 [N, K], s_w fp32 [N], wsum int32 [N] | None)."""
    N, K = W.shape
    _need(W, "W", torch.float32, (N, K))
    _need(H, "H", torch.float64, (K, K))
    q = _out(q, "q", torch.int8, (N, K), W.device)
    s_w = _out(s_w, "s_w", torch.float32, (N,), W.device)
    if want_wsum or wsum is not None:
        wsum = _out(wsum, "wsum", torch.int32, (N,), W.device)
    nbytes = q8_workspace_bytes(Q8_OP_GPTQ_INT8, 0, N, K, int(block))
    workspace, wsb = _workspace(workspace, nbytes, W.device)
    _check(_lib().q8_gptq_int8(_ptr(W), _ptr(H), N, K, float(damp), int(block), _ptr(q),
                               _ptr(s_w), _ptr(wsum), _ptr(workspace), wsb, _stream(stream)),
           "q8_gptq_int8")
    return q, s_w, wsum


def q8_linear_dq8ca_q4gsw(x: torch.Tensor, q4: torch.Tensor, gs: torch.Tensor, G: int, y=None,
                          workspace=None, stream=None) -> torch.Tensor:
    """8da4w: dynamic per-row int8 activations x int4 group weights; bf16 in, fp32 out."""
    M, K = x.shape
    N = q4.shape[0]
    _need(x, "x", torch.bfloat16, (M, K))
    _need(q4, "q4", torch.uint8, (N, K // 2))
    _need(gs, "gs", torch.float32, (N, K // G))
    y = _out(y, "y", torch.float32, (M, N), x.device)
    nbytes = q8_workspace_bytes(Q8_OP_LINEAR_DQ8CA_Q4GSW, M, N, K, G)
    workspace, wsb = _workspace(workspace, nbytes, x.device)
    _check(_lib().q8_linear_dq8ca_q4gsw(_ptr(x), _ptr(q4), _ptr(gs), int(G), _ptr(y), M, N, K,
                                        _ptr(workspace), wsb, _stream(stream)),
           "q8_linear_dq8ca_q4gsw")
    return y


def q8_gemm_s8s8_s32(a: torch.Tensor, b: torch.Tensor, acc=None, stream=None) -> torch.Tensor:
    """acc[m,n] = sum_k a[m,k] b[n,k]; int8 in, int32 out (exact)."""
    M, K = a.shape
    N = b.shape[0]
    _need(a, "a", torch.int8, (M, K))
    _need(b, "b", torch.int8, (N, K))
    acc = _out(acc, "acc", torch.int32, (M, N), a.device)
    _check(_lib().q8_gemm_s8s8_s32(_ptr(a), _ptr(b), _ptr(acc), M, N, K, _stream(stream)),
           "q8_gemm_s8s8_s32")
    return acc


def q8_selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    """Run the bounded-wait self-test kernel; returns the kernel's result flag (0: the
    wait expired as intended).  Read q8_last_device_status() afterwards."""
    res = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check(_lib().q8_selftest_bounded_wait(int(limit_ns), _ptr(res), _stream(stream)),
           "q8_selftest_bounded_wait")
    return int(res.item())


def q8_last_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(_lib().q8_last_device_status(_stream(stream)))
