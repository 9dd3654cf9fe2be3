"""GPU parity: the CUDA path (called through the C ABI) against the CPU oracle on the same
seeded inputs.  Integer stages (codes, scales, zero points, code sums) must be bit-exact;
float outputs within the tolerances in tests/tolerance.py."""
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


# ------------------------------------------------------------------ failure detection


def test_bounded_wait_reports_and_context_survives():
    """A barrier nobody completes: the bounded wait gives up after its limit, the host reads
    Q8_ERR_DEVICE, the status clears, and the next kernel runs normally."""
    assert q8.q8_last_device_status() == q8.Q8_OK
    t0 = __import__("time").time()
    assert q8.q8_selftest_bounded_wait(20_000_000) == 0       # 20 ms limit
    assert q8.q8_last_device_status() == q8.Q8_ERR_DEVICE
    assert __import__("time").time() - t0 < 10.0
    assert q8.q8_last_device_status() == q8.Q8_OK              # read-and-clear
    W = wl.weight(64, 128, seed=5)
    q, s, _ = q8.q8_quantize_weight(W.to(DEV))
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    assert np.array_equal(q.cpu().numpy(), rq)


# ------------------------------------------------------------------- weight codes (a1)


@pytest.mark.parametrize("N,K,zero_rows", [(256, 512, (7,)), (2560, 960, ()), (33, 16, (0, 32)),
                                           (11008, 4096, (5,)), (32000, 4096, ())])
def test_quantize_weight_bit_exact(N, K, zero_rows):
    W = wl.weight(N, K, seed=100 + N % 97, zero_rows=zero_rows)
    if N == 33:
        W[3] *= 1e-30
        W[4, :] = 0.0
        W[4, 5] = -2.5
    q, s, ws = q8.q8_quantize_weight(W.to(DEV))
    rq, rs, rws = oracle.quantize_weight(W.numpy())
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(ws.cpu().numpy(), rws)


def test_quantize_weight_pr1_zero_row():
    cfg = wl.PR1
    W = wl.weight(cfg["N"], cfg["K"], seed=cfg["seed"], zero_rows=cfg["zero_rows"])
    q, s, ws = q8.q8_quantize_weight(W.to(DEV))
    assert s[7].item() == 1.0 and not q[7].any().item() and ws[7].item() == 0


# ------------------------------------------------------------ activation qparams (a2)


def _edge_rows(K):
    x = wl.normal((8, K), 1.0, seed=200)
    x[1] = 0.0
    x[2] = x[2].abs()
    x[3] = -x[3].abs()
    x[4] *= 1e4
    x[5] *= 1e-30
    x[6, :] = 0.0
    x[6, 3] = 5.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("M,K", [(1, 4096), (64, 4096), (512, 4096), (4096, 4096), (3, 16),
                                 (8, 48)])
def test_choose_qparams_bit_exact(M, K):
    x = wl.normal_bf16((M, K), 1.0, seed=201 + M)
    if M >= 8:
        x[:8] = _edge_rows(K)
    s, z, xq = q8.q8_choose_qparams(x.to(DEV))
    rs, rz, rxq = oracle.choose_qparams(wl.bf16_bits(x))
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(z.cpu().numpy(), rz)
    assert np.array_equal(xq.cpu().numpy(), rxq)


def test_choose_qparams_without_codes():
    x = wl.normal_bf16((5, 64), 2.0, seed=202)
    s, z, xq = q8.q8_choose_qparams(x.to(DEV), want_codes=False)
    rs, rz, _ = oracle.choose_qparams(wl.bf16_bits(x), want_codes=False)
    assert xq is None
    assert np.array_equal(s.cpu().numpy(), rs) and np.array_equal(z.cpu().numpy(), rz)


# --------------------------------------------------------- static activation codes (a3)


def _w8a8_qparams(K):
    x, calib = wl.w8a8_inputs(1, K=K)
    mm = torch.empty(2, device=DEV)
    q8.q8_observe_minmax(calib.to(DEV), mm, reset=True)
    mn, mx = mm.cpu().tolist()
    assert (mn, mx) == oracle.minmax(calib.numpy())
    first = q8.q8_qparams_from_minmax(mn, mx)
    assert first == oracle.qparams_from_minmax(mn, mx)
    second = (float(np.float32(first[0]) / np.float32(255.0)), 0)
    return first, second


@pytest.mark.parametrize("M,K", [(1, 960), (256, 960), (2048, 960), (7, 4096), (4096, 16)])
@pytest.mark.parametrize("two", [False, True])
def test_quantize_static_bit_exact(M, K, two):
    first, second = _w8a8_qparams(K)
    x, _ = wl.w8a8_inputs(M, K=K)
    x[0, :4] = torch.tensor([1e30, -1e30, 0.0, -0.0])       # saturation and signed zero
    xq1, xq2 = q8.q8_quantize_static(x.to(DEV), first, second if two else None)
    r1, r2 = oracle.static_quant(x.numpy(), first, second if two else None)
    assert np.array_equal(xq1.cpu().numpy(), r1)
    if two:
        assert np.array_equal(xq2.cpu().numpy(), r2)


def test_observe_minmax_accumulates():
    a = wl.normal((1000,), 1.0, seed=203)
    b = wl.normal((77,), 5.0, seed=204)
    mm = torch.empty(2, device=DEV)
    q8.q8_observe_minmax(a.to(DEV), mm, reset=True)
    q8.q8_observe_minmax(b.to(DEV), mm)
    both = torch.cat([a, b]).numpy()
    assert mm.cpu().tolist() == [float(both.min()), float(both.max())]


# -------------------------------------------------------------- int4 group codes


@pytest.mark.parametrize("N,K,G", [(11008, 4096, 32), (11008, 4096, 128), (19, 256, 64),
                                   (7, 512, 256), (5, 65024, 32), (3, 2048, 256)])
def test_quantize_weight_q4gs_bit_exact(N, K, G):
    """Codes, group scales and the zero-point fold c, bit for bit; 65024 / 32 = 2032 groups
    per row exercise the fold's long fp64 chain across many 32-group rounds."""
    W = wl.weight(N, K, seed=300 + G)
    W[0, :G] = 0.0                                          # a zero group
    W[1, G:3 * G] *= 1e-20                                  # groups far smaller than the rest
    q4, gs = q8.q8_quantize_weight_q4gs(W.to(DEV), G)
    rq4, rgs = oracle.quantize_weight_q4gs(W.numpy(), G)
    assert np.array_equal(q4.cpu().numpy(), rq4)
    assert np.array_equal(gs.cpu().numpy().view(np.uint32), rgs.view(np.uint32))
    q4b, gsb, c = q8.q8_quantize_weight_q4gs(W.to(DEV), G, want_c=True)
    assert torch.equal(q4b, q4) and torch.equal(gsb, gs)
    rc = oracle.q4gs_zero_fold(rq4, rgs, G)
    assert np.array_equal(c.cpu().numpy().view(np.uint32), rc.view(np.uint32))


# ---------------------------------------------------------------------- W8A16 (a4)


def _w8a16_case(M, N, K, seed_w, seed_x, out_dtype, zero_rows=()):
    W = wl.weight(N, K, seed=seed_w, zero_rows=zero_rows)
    x = wl.normal_bf16((M, K), 1.0, seed=seed_x)
    q, s, _ = q8.q8_quantize_weight(W.to(DEV), want_wsum=False)
    y = q8.q8_linear_w8a16(x.to(DEV), q, s, out_dtype=out_dtype)
    torch.cuda.synchronize()
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    y64, absum = oracle.linear_w8a16(wl.bf16_bits(x), rq, rs)
    return y, y64, absum


def test_w8a16_pr1_fp32():
    c = wl.PR1
    y, y64, absum = _w8a16_case(c["M"], c["N"], c["K"], c["seed"], c["seed"] + 1000,
                                torch.float32, zero_rows=c["zero_rows"])
    check_f32(y.cpu().numpy(), y64, absum, "PR1")
    assert (y[:, 7] == 0).all()


@pytest.mark.parametrize("shape", wl.W8A16_SWEEP_SHAPES, ids=lambda s: f"K{s.K}xN{s.N}")
@pytest.mark.parametrize("M", wl.W8A16_SWEEP_M)
def test_w8a16_sweep_bf16(shape, M):
    y, y64, absum = _w8a16_case(M, shape.N, shape.K, wl.W8A16_SWEEP_SEED_W,
                                wl.W8A16_SWEEP_SEED_X, torch.bfloat16)
    check_bf16(_bits(y), y64, absum, f"W8A16 M={M} K={shape.K} N={shape.N}")


@pytest.mark.parametrize("M,N,K", [
    # TMA-streamed path (K % 64 == 0, M <= 16): ragged N, K not a multiple of the 1 KB stage
    (16, 1, 64), (1, 17, 64), (5, 2049, 1024), (12, 1000, 4160), (9, 33, 128), (2, 300, 11008),
    # ... activations at the tensor-memory limit (512 columns), and past it in shared memory
    (16, 100, 8192), (8, 50, 16384), (1, 70, 16448), (3, 33, 17472),
    # ... 2 KB stages (K % 2048 == 0, long streams per CTA), ragged N
    (3, 9000, 4096), (16, 20000, 6144), (1, 40000, 8192),
    # register-streamed fallback (K % 64 != 0, or M > 16)
    (3, 17, 16), (9, 40, 48), (17, 33, 80), (40, 130, 1040), (5, 2049, 2000)])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_w8a16_ragged(M, N, K, out):
    y, y64, absum = _w8a16_case(M, N, K, 400 + N, 401 + M, out)
    if out == torch.float32:
        check_f32(y.cpu().numpy(), y64, absum, "ragged")
    else:
        check_bf16(_bits(y), y64, absum, "ragged")


def _w8a16_direct(x_bf16, W, out_dtype=torch.float32):
    q, s, _ = q8.q8_quantize_weight(W.to(DEV), want_wsum=False)
    y = q8.q8_linear_w8a16(x_bf16.to(DEV), q, s, out_dtype=out_dtype)
    torch.cuda.synchronize()
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    y64, absum = oracle.linear_w8a16(wl.bf16_bits(x_bf16), rq, rs)
    return y.cpu().numpy(), y64, absum


def _range_edge_rows(M, K, e_small, seed):
    """Row 0..M-1: x[:, 0] = 2^10 with an all-zero weight column (so it only sets the row's
    exponent range), every other element +-(1 + j/128) * 2^e_small.  The output is then the
    sum of the small elements alone, and the tolerance is relative to it."""
    g = torch.Generator().manual_seed(seed)
    sign = torch.where(torch.rand(M, K, generator=g) < 0.5, -1.0, 1.0)
    frac = 1.0 + torch.randint(0, 128, (M, K), generator=g).to(torch.float32) / 128.0
    x = sign * frac * 2.0 ** e_small
    x[:, 0] = 1024.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("M,N", [(16, 2000), (4, 32000)])
@pytest.mark.parametrize("e_small", [-22, -23])
def test_w8a16_wide_row_range(M, N, e_small):
    """Rows whose elements span 32-33 binades (one 2^10 element on an all-zero weight
    column, the rest near 2^-22 or 2^-23): the bf16 operands carry every element exactly,
    so the output -- the small elements' sum alone -- must hold to fp32 rounding."""
    K = 4096
    x = _range_edge_rows(M, K, e_small, seed=90 + M)
    W = wl.weight(N, K, seed=91)
    W[:, 0] = 0.0
    y, y64, absum = _w8a16_direct(x, W)
    check_f32(y, y64, absum, f"range boundary 2^{e_small}")


@pytest.mark.parametrize("M,N", [(16, 1000), (4, 32000)])
@pytest.mark.parametrize("kind", ["wide", "tiny", "inf"])
def test_w8a16_activation_ranges(M, N, kind):
    """Extreme activation rows: exponents spread over 2^-120..2^60, values near the bf16
    subnormal range, and rows holding inf / NaN (which must propagate as in IEEE)."""
    K = 4096
    g = torch.Generator().manual_seed(95)
    x = torch.randn(M, K, generator=g, dtype=torch.float64)
    if kind == "wide":
        x = x * torch.pow(2.0, torch.randint(-120, 61, (M, K), generator=g).to(torch.float64))
    elif kind == "tiny":
        x = x * 2.0 ** -128
    x = x.to(torch.float32).to(torch.bfloat16)
    if kind == "inf":
        x[0, 3] = float("inf")
        x[1, 7] = float("nan")
    W = wl.weight(N, K, seed=96)
    y, y64, absum = _w8a16_direct(x, W)
    if kind == "inf":
        y = y.astype(np.float64)
        assert np.array_equal(np.isnan(y), np.isnan(y64))
        assert np.array_equal(np.isinf(y), np.isinf(y64))
        fin = np.isfinite(y64)
        check_f32(y[fin], y64[fin], absum[fin], "finite rows")
    else:
        check_f32(y, y64, absum, kind)


def test_w8a16_empty_m():
    q = torch.zeros(16, 64, dtype=torch.int8, device=DEV)
    s = torch.ones(16, device=DEV)
    y = q8.q8_linear_w8a16(torch.zeros(0, 64, dtype=torch.bfloat16, device=DEV), q, s)
    assert y.shape == (0, 16)


# ----------------------------------------------------------------------- W8A8 (a5/a6)


@pytest.mark.parametrize("M", [1, 5, 16, 37])
@pytest.mark.parametrize("N", wl.W8A8_N)
@pytest.mark.parametrize("two", [False, True])
def test_w8a8_small_m(M, N, two):
    K = wl.W8A8_K
    first, second = _w8a8_qparams(K)
    x, _ = wl.w8a8_inputs(M, K=K)
    W = wl.weight(N, K, seed=wl.W8A8_SEED_W)
    q, s, ws = q8.q8_quantize_weight(W.to(DEV))
    y = q8.q8_linear_w8a8(x.to(DEV), first, q, ws, s, second=second if two else None)
    torch.cuda.synchronize()
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    y64, absum, _, _ = oracle.linear_w8a8(x.numpy(), first, rq, rs,
                                          second=second if two else None)
    check_f32(y.cpu().numpy(), y64, absum, f"W8A8 M={M} N={N} two={two}")


@pytest.mark.parametrize("M,N,K,rows", [
    (128, 256, 128, None), (256, 512, 1024, None), (300, 300, 960, None), (37, 33, 128, None),
    (17, 2560, 960, None), (1000, 1000, 4096, None),
    (4096, 4096, 4096, [0, 1, 127, 128, 1000, 2047, 4095]),
    (4096, 11008, 4096, [0, 129, 4095]), (4096, 4096, 11008, [5, 2100, 4094])])
def test_gemm_s8s8_s32_bit_exact(M, N, K, rows):
    """int32 accumulators of the tcgen05 int8 GEMM, bit for bit (sampled rows at full size)."""
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    a = torch.randint(-128, 128, (M, K), dtype=torch.int8, generator=g)
    b = torch.randint(-128, 128, (N, K), dtype=torch.int8, generator=g)
    acc = q8.q8_gemm_s8s8_s32(a.to(DEV), b.to(DEV)).cpu().numpy()
    ref = oracle.gemm_s8s8_s32(a.numpy(), b.numpy(), rows=rows)
    got = acc if rows is None else acc[rows]
    assert np.array_equal(got, ref)


def test_gemm_s8s8_s32_extreme_values():
    """All-(-128) operands: the largest magnitude sums (K * 2^14) stay exact in int32."""
    M, N, K = 130, 260, 4096
    a = torch.full((M, K), -128, dtype=torch.int8)
    b = torch.full((N, K), -128, dtype=torch.int8)
    acc = q8.q8_gemm_s8s8_s32(a.to(DEV), b.to(DEV)).cpu().numpy()
    assert (acc == K * 128 * 128).all()


@pytest.mark.parametrize("M", [256, 2048])
@pytest.mark.parametrize("N", wl.W8A8_N)
@pytest.mark.parametrize("two", [False, True])
def test_w8a8_prefill_tensor_core(M, N, two):
    """Static W8A8 at K = 960 on the tensor-core path (single and two-pass)."""
    K = wl.W8A8_K
    first, second = _w8a8_qparams(K)
    x, _ = wl.w8a8_inputs(M, K=K)
    W = wl.weight(N, K, seed=wl.W8A8_SEED_W)
    q, s, ws = q8.q8_quantize_weight(W.to(DEV))
    y = q8.q8_linear_w8a8(x.to(DEV), first, q, ws, s, second=second if two else None)
    torch.cuda.synchronize()
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    y64, absum, _, _ = oracle.linear_w8a8(x.numpy(), first, rq, rs,
                                          second=second if two else None)
    check_f32(y.cpu().numpy(), y64, absum, f"W8A8 TC M={M} N={N} two={two}")


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 11008), (11008, 4096)])
@pytest.mark.parametrize("two", [False, True])
def test_w8a8_llama_prefill_sampled(K, N, two):
    """Llama-shaped prefill linears at M = 4096 (sampled output rows vs the oracle)."""
    M = wl.LLAMA_PREFILL_M
    x = wl.normal((M, K), 1.0, seed=500 + K + N)
    mm = torch.empty(2, device=DEV)
    q8.q8_observe_minmax(x.to(DEV), mm, reset=True)
    first = q8.q8_qparams_from_minmax(*mm.cpu().tolist())
    second = (float(np.float32(first[0]) / np.float32(255.0)), 0) if two else None
    W = wl.weight(N, K, seed=600 + K + N)
    q, s, ws = q8.q8_quantize_weight(W.to(DEV))
    y = q8.q8_linear_w8a8(x.to(DEV), first, q, ws, s, second=second)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 2049, M - 1]
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    y64, absum, _, _ = oracle.linear_w8a8(x.numpy(), first, rq, rs, second=second, rows=rows)
    check_f32(y.cpu().numpy()[rows], y64, absum, f"W8A8 llama K={K} N={N} two={two}")


@pytest.mark.parametrize("M,N,K", [(1, 32000, 4096), (16, 11008, 4096), (4, 2560, 960)])
def test_w8a16_repeat_bit_identical(M, N, K):
    """The warps' partial sums are added in a fixed order (no float atomics), so repeated
    calls give the same bits (wide and narrow stages, 1 and 2 activation tiles)."""
    W = wl.weight(N, K, seed=880 + M)
    x = wl.normal_bf16((M, K), 1.0, seed=881 + M).to(DEV)
    q, s, _ = q8.q8_quantize_weight(W.to(DEV), want_wsum=False)
    ref = q8.q8_linear_w8a16(x, q, s, out_dtype=torch.float32).cpu()
    for _ in range(5):
        y = q8.q8_linear_w8a16(x, q, s, out_dtype=torch.float32).cpu()
        assert torch.equal(y.view(torch.int32), ref.view(torch.int32))


@pytest.mark.parametrize("M,G", [(1, 128), (8, 32), (16, 64), (40, 64)])
def test_dq8ca_decode_repeat_bit_identical(M, G):
    """The 8da4w decode stream is deterministic too (fixed-order partial sums), and so is
    the K-split of the small-M GEMM (the last part adds all parts in part order)."""
    N, K = 11008, 4096
    W = wl.weight(N, K, seed=890 + M)
    x = wl.normal_bf16((M, K), 1.0, seed=891 + M).to(DEV)
    q4, gs = q8.q8_quantize_weight_q4gs(W.to(DEV), G)
    ref = q8.q8_linear_dq8ca_q4gsw(x, q4, gs, G).cpu()
    for _ in range(5):
        y = q8.q8_linear_dq8ca_q4gsw(x, q4, gs, G).cpu()
        assert torch.equal(y.view(torch.int32), ref.view(torch.int32))


# ----------------------------------------------------------------------- 8da4w (a7)


def _q4_case(M, N, K, G, seed_x, seed_w, zero_x_rows=()):
    x = wl.normal_bf16((M, K), 1.0, seed=seed_x)
    for r in zero_x_rows:
        x[r] = 0
    W = wl.weight(N, K, seed=seed_w)
    q4, gs = q8.q8_quantize_weight_q4gs(W.to(DEV), G)
    y = q8.q8_linear_dq8ca_q4gsw(x.to(DEV), q4, gs, G)
    torch.cuda.synchronize()
    return x, q4.cpu().numpy(), gs.cpu().numpy(), y.cpu().numpy()


@pytest.mark.parametrize("M", wl.Q4_M)
@pytest.mark.parametrize("G", wl.Q4_G)
def test_dq8ca_q4gsw_config(M, G):
    """8da4w at K = 4096, N = 11008 (sampled rows for the large M)."""
    K, N = wl.Q4_K, wl.Q4_N
    x, q4, gs, y = _q4_case(M, N, K, G, wl.Q4_SEED_X, wl.Q4_SEED_W, zero_x_rows=(0,))
    rows = None if M <= 64 else [0, 1, 63, 64, M // 2, M - 1]
    s, z, xq = oracle.choose_qparams(wl.bf16_bits(x))
    y64, absum = oracle.linear_dq8ca_q4gsw(xq, s, z, q4, gs, G, rows=rows)
    got = y if rows is None else y[rows]
    check_f32(got, y64, absum, f"8da4w M={M} G={G}")
    assert (y[0] == 0).all()                    # an all-zero activation row gives 0 exactly


@pytest.mark.parametrize("M,N,K,G", [(3, 17, 128, 32), (9, 40, 256, 64), (17, 33, 512, 128),
                                     (5, 300, 1024, 256), (1, 1, 128, 128), (70, 129, 384, 32),
                                     # the TMA stream: partial last stage, ragged N, 9..16 rows
                                     (2, 1000, 2176, 32), (16, 4097, 4096, 128),
                                     (8, 2000, 6144, 64), (12, 700, 4224, 32), (4, 11008, 4096, 256),
                                     # rows longer than the stream keeps in registers
                                     (1, 300, 12288, 64), (3, 500, 10240, 128),
                                     # above 64 rows, ragged last tiles and odd N: the bf16
                                     # GEMM (G <= 64; 256-row tiles from 2048 rows) and the
                                     # int8 one (G = 256; G = 128 below 2048 rows)
                                     (2100, 300, 512, 64), (600, 18500, 256, 64),
                                     (2048, 129, 256, 256), (300, 19000, 512, 256),
                                     (150, 5000, 1024, 128),
                                     # 17..64 rows: the GEMM expands the int4 codes itself
                                     (33, 1000, 2176, 64), (64, 300, 4096, 256),
                                     (20, 129, 128, 32), (50, 257, 1024, 128)])
def test_dq8ca_q4gsw_ragged(M, N, K, G):
    x, q4, gs, y = _q4_case(M, N, K, G, 900 + M, 901 + N)
    s, z, xq = oracle.choose_qparams(wl.bf16_bits(x))
    y64, absum = oracle.linear_dq8ca_q4gsw(xq, s, z, q4, gs, G)
    check_f32(y, y64, absum, f"8da4w ragged M={M} N={N} K={K} G={G}")


@pytest.mark.parametrize("M,K,G", [(1, 4096, 32), (2, 12288, 128), (7, 2176, 64), (16, 4096, 256)])
def test_dq8ca_decode_workspace_codes(M, K, G):
    """Up to 16 rows the decode stream quantizes the activations inside the kernel; the
    workspace still receives them (codes [M, K] at offset 0, then the scales and the zero
    points, each on a 256-byte boundary) and they are the oracle's choose_qparams bit for
    bit, including an all-zero row and a row with a single huge value."""
    N = 300
    x = wl.normal_bf16((M, K), 1.0, seed=4300 + M)
    x[0] = 0
    if M > 1:
        x[M - 1, K // 3] = 3.0e4
    W = wl.weight(N, K, seed=4301)
    q4, gs = q8.q8_quantize_weight_q4gs(W.to(DEV), G)
    nb = q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_DQ8CA_Q4GSW, M, N, K, G)
    work = torch.full((nb,), 0x5A, dtype=torch.uint8, device=DEV)
    q8.q8_linear_dq8ca_q4gsw(x.to(DEV), q4, gs, G, workspace=work)
    torch.cuda.synchronize()
    w = work.cpu().numpy()
    rs, rz, rxq = oracle.choose_qparams(wl.bf16_bits(x))
    off_s = -(-M * K // 256) * 256
    off_z = off_s + -(-M * 4 // 256) * 256
    assert np.array_equal(w[:M * K].view(np.int8).reshape(M, K), rxq)
    assert np.array_equal(w[off_s:off_s + 4 * M].view(np.float32), np.asarray(rs, np.float32))
    assert np.array_equal(w[off_z:off_z + 4 * M].view(np.int32), np.asarray(rz, np.int32))


@pytest.mark.parametrize("M,K", [(300, 256), (5, 256), (16, 4096), (1, 12288), (3, 2304),
                                 (40, 512), (65, 768), (1000, 1024)])
def test_dq8ca_group_partials_exact(M, K):
    """Unit group scales: y / s must be the exact integer sum_k (xq - z) q4 (one fp32
    rounding of s * T).  Above 64 rows this is the int8 tensor-core GEMM (its zero-point term
    and int32 -> fp32 steps must be exact), 17..64 rows the bf16 one with the int4 -> bf16
    expansion inside; up to 16 rows the decode stream, whose in-kernel activation codes and
    zero points must then be the oracle's bit for bit."""
    N, G = 200, 256
    g = torch.Generator().manual_seed(4242)
    x = wl.normal_bf16((M, K), 1.0, seed=4243 + M)
    q4 = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, generator=g)   # any nibbles
    gs = torch.ones(N, K // G)
    y = q8.q8_linear_dq8ca_q4gsw(x.to(DEV), q4.to(DEV), gs.to(DEV), G).cpu().numpy()
    s, z, xq = oracle.choose_qparams(wl.bf16_bits(x))
    lo = (q4.numpy() & 0xF).astype(np.int64)
    hi = (q4.numpy() >> 4).astype(np.int64)
    codes = np.empty((N, K), np.int64)
    codes[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    codes[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    T = (xq.astype(np.int64) - z[:, None]) @ codes.T
    assert np.abs(T).max() < 2 ** 24
    want = s.astype(np.float32)[:, None] * T.astype(np.float32)      # one fp32 rounding
    assert np.array_equal(y, want)
