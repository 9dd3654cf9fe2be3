"""GPU parity of the weight-grid option and the bias epilogues against the oracle.

* q8_quantize_weight(grid="full128"): weight_int8 of the SmolVLM q8 page (observer scale
  amax/127.5 floored at fp32 eps, codes -128..127) -- codes, scales and code sums bit-exact.
* bias: Int8Linear (ROCm INT8 page) adds an optional [out] bias after the scaled matmul;
  Q8Linear (SmolVLM q8 page) adds it to the first pass only.  Every kernel behind
  q8_linear_w8a16 and q8_linear_w8a8 (TMA stream, GEMV fallback, tensor-core GEMM) is
  covered, with weights of both grids."""
import numpy as np
import pytest
import torch

import int8_quantized_linear_q8_b200 as q8
import oracle
import q8_workloads as wl
from int8_quantized_linear_q8_b200 import build as q8build
from tolerance import check_bf16, check_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q8build.build()
    q8.lib()
    yield
    assert q8.q8_last_device_status() == q8.Q8_OK


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _full128_weight(N, K, seed):
    """Seeded weight with the grid's corner cases: an all-zero row, a row below the eps
    floor, and rows whose extreme is negative (codes -128 or -127, depending on how
    amax/127.5 rounds in fp32)."""
    W = wl.weight(N, K, seed=seed)
    if N > 3:
        W[1] = 0.0
        W[2] *= 1e-9
        W[3:, 0] = -W[3:].abs().amax(dim=1) * 1.01
    return W


@pytest.mark.parametrize("N,K", [(256, 512), (2560, 960), (33, 16), (11008, 4096),
                                 (32000, 4096)])
def test_quantize_weight_full128_bit_exact(N, K):
    W = _full128_weight(N, K, seed=700 + N % 97)
    q, s, ws = q8.q8_quantize_weight(W.to(DEV), grid="full128")
    rq, rs, rws = oracle.quantize_weight(W.numpy(), grid="full128")
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(ws.cpu().numpy(), rws)
    if N > 3:
        assert (rq[3:, 0] == -128).any()             # the case exists at these sizes


def test_quantize_weight_full128_golden_rows():
    """The hand-worked rows of tests/golden/weight_int8_full128_rows.txt, on the GPU."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "weight_int8_full128_rows.txt")
    rows = []
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append([p.split() for p in line.split("|")])
    W = torch.tensor([[float(v) for v in r[0]] for r in rows], dtype=torch.float32)
    W = torch.cat([W, torch.zeros(len(rows), 8)], dim=1)     # K = 16
    q, s, ws = q8.q8_quantize_weight(W.to(DEV), grid="full128")
    for i, r in enumerate(rows):
        assert q[i, :8].cpu().tolist() == [int(v) for v in r[2]], f"row {i}"
        assert s[i].item() == np.float32(float(r[1][0])), f"row {i} scale"
        assert ws[i].item() == int(r[3][0]), f"row {i} sum"


def _bias(N, seed):
    return wl.normal((N,), 0.5, seed=seed)


@pytest.mark.parametrize("M,N,K", [
    (1, 2560, 960), (4, 11008, 4096), (16, 32000, 4096),     # TMA stream (sweep shapes)
    (3, 2049, 1024), (16, 100, 8192), (1, 40000, 8192),      # ragged N, 2 KB stages
    (17, 33, 80), (40, 130, 1040), (5, 2049, 2000)])         # GEMV fallback
@pytest.mark.parametrize("grid", ["sym127", "full128"])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_w8a16_bias(M, N, K, grid, out):
    W = _full128_weight(N, K, seed=710 + N % 31) if grid == "full128" else \
        wl.weight(N, K, seed=710 + N % 31)
    x = wl.normal_bf16((M, K), 1.0, seed=711 + M)
    b = _bias(N, 712 + N % 7)
    q, s, _ = q8.q8_quantize_weight(W.to(DEV), want_wsum=False, grid=grid)
    y = q8.q8_linear_w8a16(x.to(DEV), q, s, out_dtype=out, bias=b.to(DEV))
    torch.cuda.synchronize()
    rq, rs, _ = oracle.quantize_weight(W.numpy(), grid=grid)
    y64, absum = oracle.linear_w8a16(wl.bf16_bits(x), rq, rs, bias=b.numpy())
    what = f"W8A16 bias M={M} N={N} K={K} {grid}"
    if out == torch.float32:
        check_f32(y.cpu().numpy(), y64, absum, what)
    else:
        check_bf16(_bits(y), y64, absum, what)


def _w8a8_qparams(K):
    x, calib = wl.w8a8_inputs(1, K=K)
    first = oracle.qparams_from_minmax(*oracle.minmax(calib.numpy()))
    second = (float(np.float32(first[0]) / np.float32(255.0)), 0)
    return first, second


@pytest.mark.parametrize("M", [1, 16, 37, 256, 2048])       # GEMV and tensor-core paths
@pytest.mark.parametrize("N", [960, 2560])
@pytest.mark.parametrize("two", [False, True])
@pytest.mark.parametrize("grid", ["sym127", "full128"])
def test_w8a8_bias(M, N, two, grid):
    K = wl.W8A8_K
    first, second = _w8a8_qparams(K)
    x, _ = wl.w8a8_inputs(M, K=K)
    W = _full128_weight(N, K, seed=720) if grid == "full128" else wl.weight(N, K, seed=720)
    b = _bias(N, 721)
    q, s, ws = q8.q8_quantize_weight(W.to(DEV), grid=grid)
    y = q8.q8_linear_w8a8(x.to(DEV), first, q, ws, s, second=second if two else None,
                          bias=b.to(DEV))
    torch.cuda.synchronize()
    rq, rs, _ = oracle.quantize_weight(W.numpy(), grid=grid)
    y64, absum, _, _ = oracle.linear_w8a8(x.numpy(), first, rq, rs,
                                          second=second if two else None, bias=b.numpy())
    check_f32(y.cpu().numpy(), y64, absum, f"W8A8 bias M={M} N={N} two={two} {grid}")


def test_w8a8_bias_llama_prefill_sampled():
    """The tensor-core GEMM at a Llama prefill shape (M = 4096), bias in the epilogue,
    checked on sampled rows (the oracle computes only those)."""
    M, N, K = 4096, 11008, 4096
    x, calib = wl.w8a8_inputs(M, K=K)
    first = oracle.qparams_from_minmax(*oracle.minmax(calib.numpy()))
    W = wl.weight(N, K, seed=730)
    b = _bias(N, 731)
    q, s, ws = q8.q8_quantize_weight(W.to(DEV))
    y = q8.q8_linear_w8a8(x.to(DEV), first, q, ws, s, bias=b.to(DEV))
    torch.cuda.synchronize()
    rows = [0, 127, 128, 2049, 4095]
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    y64, absum, _, _ = oracle.linear_w8a8(x.numpy(), first, rq, rs, rows=rows, bias=b.numpy())
    check_f32(y.cpu().numpy()[rows], y64, absum, "W8A8 bias 4096x11008x4096")


def test_bias_none_is_bit_identical_to_plain_call():
    """bias=None goes through the plain entry points; a zero bias gives the same values."""
    M, N, K = 4, 11008, 4096
    W = wl.weight(N, K, seed=740)
    x = wl.normal_bf16((M, K), 1.0, seed=741).to(DEV)
    q, s, _ = q8.q8_quantize_weight(W.to(DEV), want_wsum=False)
    y0 = q8.q8_linear_w8a16(x, q, s, out_dtype=torch.float32)
    yz = q8.q8_linear_w8a16(x, q, s, out_dtype=torch.float32,
                            bias=torch.zeros(N, device=DEV))
    assert torch.equal(y0, yz)


# ------------------------------------------- residual calibration observer (f2)


@pytest.mark.parametrize("chunks", [[1], [4096 * 960], [1000, 3, 4097, 250000], [960] * 9])
def test_observe_residual_minmax_bit_exact(chunks):
    """The second calibration run's observer (x - fake_quant(x, first)) over a stream of
    chunks: reset on the first, then accumulate; min and max bit-exact against the oracle."""
    first = (float(np.float32(0.0625)), -3)
    xs = [wl.normal((n,), 2.0, seed=750 + i).numpy() for i, n in enumerate(chunks)]
    xs[0][0] = 1e4                                      # clamped at 127
    xs[-1][-1] = -1e4                                   # clamped at -128
    mm = torch.empty(2, device=DEV)
    for i, x in enumerate(xs):
        q8.q8_observe_residual_minmax(torch.from_numpy(x).to(DEV), first, mm, reset=(i == 0))
    got = tuple(mm.cpu().tolist())
    assert got == oracle.residual_minmax(np.concatenate(xs), first)


def test_two_pass_calibration_chain():
    """calibrate with two passes (SmolVLM q8 page) end to end on the GPU: observe the
    calibration draw -> (s1, z1); observe its first-pass errors -> (s2, z2); both equal the
    oracle's; then the two-pass W8A8 linear with those qparams matches the oracle."""
    K, N, M = wl.W8A8_K, 2560, 37
    x, calib = wl.w8a8_inputs(M, K=K)
    mm = torch.empty(2, device=DEV)
    q8.q8_observe_minmax(calib.to(DEV), mm, reset=True)
    first = q8.q8_qparams_from_minmax(*mm.cpu().tolist())
    assert first == oracle.qparams_from_minmax(*oracle.minmax(calib.numpy()))
    q8.q8_observe_residual_minmax(calib.to(DEV), first, mm, reset=True)
    rmin, rmax = mm.cpu().tolist()
    assert (rmin, rmax) == oracle.residual_minmax(calib.numpy(), first)
    second = q8.q8_qparams_from_minmax(rmin, rmax)
    assert second == oracle.qparams_from_minmax(rmin, rmax)
    W = wl.weight(N, K, seed=760)
    q, s, ws = q8.q8_quantize_weight(W.to(DEV))
    for xm in (x, calib[:2048]):
        y = q8.q8_linear_w8a8(xm.to(DEV), first, q, ws, s, second=second)
        torch.cuda.synchronize()
        rq, rs, _ = oracle.quantize_weight(W.numpy())
        y64, absum, _, _ = oracle.linear_w8a8(xm.numpy(), first, rq, rs, second=second)
        check_f32(y.cpu().numpy(), y64, absum, f"calibrated two-pass M={xm.shape[0]}")
