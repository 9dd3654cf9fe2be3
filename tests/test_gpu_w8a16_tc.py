"""GPU parity of q8_linear_w8a16_planes -- W8A16 on the int8 tensor cores over exact digit planes
of the activations -- against the oracle.  Besides the contract tolerances of tests/tolerance.py,
fp32 outputs are held to about one rounding of the exact dot product, which is what the
digit-plane recombination gives."""
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


_WS = {}


def _ws(M, N, K):
    """One zero-filled workspace for the module, grown as needed (flags persist across calls)."""
    n = q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A16_PLANES, M, N, K)
    if n == 0:
        return None
    if "ws" not in _WS or _WS["ws"].numel() < n:
        _WS["ws"] = torch.zeros(n, dtype=torch.uint8, device=DEV)
    return _WS["ws"]


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _tight(y, y64, absum, what):
    """fp32 output within one rounding (plus slack for the oracle's own fp64 sum)."""
    y = np.asarray(y, np.float64)
    bound = 2.0 ** -24 * np.abs(y64) * (1 + 1e-6) + 1e-12 * absum + 1e-40
    bad = ~(np.abs(y - y64) <= bound)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} outputs beyond one rounding; first at {i}: "
                             f"got {y[i]!r}, oracle {y64[i]!r}")


def _case(x_bf16, W, out_dtype):
    """Run the tensor-core path and the oracle on the same bf16 activations and weight."""
    M, K = x_bf16.shape
    N = W.shape[0]
    q, s, _ = q8.q8_quantize_weight(W.to(DEV), want_wsum=False)
    y = q8.q8_linear_w8a16_planes(x_bf16.to(DEV), q, s, _ws(M, N, K), out_dtype=out_dtype)
    torch.cuda.synchronize()
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    y64, absum = oracle.linear_w8a16(wl.bf16_bits(x_bf16), rq, rs)
    return y, y64, absum


@pytest.mark.parametrize("shape", wl.W8A16_SWEEP_SHAPES, ids=lambda s: f"K{s.K}xN{s.N}")
@pytest.mark.parametrize("M", wl.W8A16_SWEEP_M)
def test_w8a16_tc_sweep(shape, M):
    W = wl.weight(shape.N, shape.K, seed=wl.W8A16_SWEEP_SEED_W)
    x = wl.normal_bf16((M, shape.K), 1.0, seed=wl.W8A16_SWEEP_SEED_X)
    y, y64, absum = _case(x, W, torch.bfloat16)
    check_bf16(_bits(y), y64, absum, f"W8A16 tc M={M} K={shape.K} N={shape.N}")
    y, y64, absum = _case(x, W, torch.float32)
    check_f32(y.cpu().numpy(), y64, absum, "sweep fp32")
    _tight(y.cpu().numpy(), y64, absum, "sweep fp32")


@pytest.mark.parametrize("M,N,K", [
    # fewer units than SMs; a tile split over many CTAs (N = 128, K = 4096: 32 CTAs, 1 unit
    # each); ragged N and K (K % 128 != 0); the largest K; M at the plane-budget breaks
    (1, 1, 16), (16, 1, 16), (3, 129, 144), (5, 2049, 1040), (9, 33, 4160), (16, 300, 11008),
    (2, 1000, 96), (16, 4097, 4096), (7, 128, 128), (1, 128, 4096), (8, 257, 8192),
    (1, 200, 65520), (4, 640, 2064), (12, 5000, 1024)])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_w8a16_tc_ragged(M, N, K, out):
    W = wl.weight(N, K, seed=700 + N % 101)
    x = wl.normal_bf16((M, K), 1.0, seed=701 + M)
    y, y64, absum = _case(x, W, out)
    if out == torch.float32:
        check_f32(y.cpu().numpy(), y64, absum, "tc ragged")
        _tight(y.cpu().numpy(), y64, absum, "tc ragged")
    else:
        check_bf16(_bits(y), y64, absum, "tc ragged")


def _wide_rows(M, K, seed):
    """Rows spanning most of the bf16 exponent range: normal values scaled by 2^e with e in
    [-125, 60], exact zeros, subnormals, and (row 1) an all-zero row."""
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(M, K, generator=g, dtype=torch.float64)
    e = torch.randint(-125, 61, (M, K), generator=g).to(torch.float64)
    x = v * torch.pow(2.0, e)
    x[:, ::7] = 0.0
    x[:, 3::11] = torch.randn(M, len(range(3, K, 11)), generator=g, dtype=torch.float64) * 2.0 ** -131
    if M > 1:
        x[1] = 0.0
    return x.to(torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_w8a16_tc_wide_range(M):
    """Exponents spread over 2^-131..2^60: one row fits 80 planes exactly; with 4 and 16 rows
    the plane budget (20 / 10) is exceeded and the smallest elements take the residual path."""
    K, N = 1024, 300
    x = _wide_rows(M, K, seed=31 + M)
    W = wl.weight(N, K, seed=32)
    y, y64, absum = _case(x, W, torch.float32)
    check_f32(y.cpu().numpy(), y64, absum, "wide range")
    _tight(y.cpu().numpy(), y64, absum, "wide range")


def test_w8a16_tc_nonfinite():
    """inf and NaN activations propagate as in IEEE arithmetic (inf * 0 = NaN)."""
    M, K, N = 4, 256, 200                     # row 3 stays finite
    x = wl.normal_bf16((M, K), 1.0, seed=41)
    x[0, 5] = float("inf")
    x[1, 9] = float("-inf")
    x[2, 17] = float("nan")
    W = wl.weight(N, K, seed=42)
    y, y64, absum = _case(x, W, torch.float32)
    y = y.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isnan(y), np.isnan(y64))
    inf = np.isinf(y64)
    assert np.array_equal(np.isinf(y), inf)
    assert np.array_equal(np.sign(y[inf]), np.sign(y64[inf]))
    fin = np.isfinite(y64)
    assert fin.sum() > 0
    _tight(y[fin], y64[fin], absum[fin], "finite entries")


def test_w8a16_tc_repeat_same_workspace():
    """Calls of different sizes alternate on one workspace (per-call flags) and repeat
    bit-identically."""
    shapes = [(1, 2560, 960), (16, 1000, 4096), (4, 129, 144)]
    ref = {}
    for rnd in range(3):
        for (M, N, K) in shapes:
            W = wl.weight(N, K, seed=50 + N % 13)
            x = wl.normal_bf16((M, K), 1.0, seed=51 + M)
            y, y64, absum = _case(x, W, torch.float32)
            yb = y.cpu().numpy()
            if rnd == 0:
                _tight(yb, y64, absum, "repeat")
                ref[(M, N, K)] = yb
            else:
                assert np.array_equal(yb, ref[(M, N, K)])


def test_w8a16_tc_workspace_checks():
    M, N, K = 4, 256, 512
    W = wl.weight(N, K, seed=60)
    q, s, _ = q8.q8_quantize_weight(W.to(DEV), want_wsum=False)
    x = wl.normal_bf16((M, K), 1.0, seed=61).to(DEV)
    need = q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A16_PLANES, M, N, K)
    assert need > 0
    small = torch.zeros(need - 1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(q8.Q8Error) as ei:
        q8.q8_linear_w8a16_planes(x, q, s, small)
    assert ei.value.status == q8.Q8_ERR_WORKSPACE
    with pytest.raises(q8.Q8Error) as ei:
        q8.q8_linear_w8a16_planes(x, q, s, None)
    assert ei.value.status == q8.Q8_ERR_WORKSPACE
    # more than 16 rows needs no workspace and runs the workspace-free path
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A16_PLANES, 17, N, K) == 0
    x17 = wl.normal_bf16((17, K), 1.0, seed=62)
    y = q8.q8_linear_w8a16_planes(x17.to(DEV), q, s, None, out_dtype=torch.float32)
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    y64, absum = oracle.linear_w8a16(wl.bf16_bits(x17), rq, rs)
    check_f32(y.cpu().numpy(), y64, absum, "M=17 fallback")


def test_w8a16_tc_graph_replay():
    """One call captured in a CUDA graph and replayed with new activations each time: the
    cross-CTA flags must belong to each replay, not to the capture, so every replay matches
    the oracle on its own inputs (tiles here span several CTAs: 64 tiles x 16 K-blocks)."""
    M, N, K = 4, 8192, 2048
    W = wl.weight(N, K, seed=70)
    q, s, _ = q8.q8_quantize_weight(W.to(DEV), want_wsum=False)
    rq, rs, _ = oracle.quantize_weight(W.numpy())
    ws = q8.q8_w8a16_planes_workspace(M, N, K, device=DEV)
    xs = torch.empty(M, K, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(M, N, dtype=torch.float32, device=DEV)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        xs.copy_(wl.normal_bf16((M, K), 1.0, seed=71).to(DEV))
        q8.q8_linear_w8a16_planes(xs, q, s, ws, y=y, out_dtype=torch.float32)   # warm
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        q8.q8_linear_w8a16_planes(xs, q, s, ws, y=y, out_dtype=torch.float32)
    for r in range(4):
        x = wl.normal_bf16((M, K), 1.0 + r, seed=72 + r)
        xs.copy_(x.to(DEV))
        y.fill_(float("nan"))
        gr.replay()
        torch.cuda.synchronize()
        y64, absum = oracle.linear_w8a16(wl.bf16_bits(x), rq, rs)
        _tight(y.cpu().numpy(), y64, absum, f"graph replay {r}")


@pytest.mark.parametrize("M", [1, 16])
def test_w8a16_tc_full_int8_grid(M):
    """Weights on the observer grid (codes down to -128, weight_int8 of the SmolVLM q8 page):
    the digit-plane products stay exact in int32 (|P| <= 127 * 128 * K)."""
    N, K = 2560, 960
    W = wl.weight(N, K, seed=80)
    W[3:, 0] = -W[3:].abs().amax(dim=1) * 1.01
    q, s, _ = q8.q8_quantize_weight(W.to(DEV), want_wsum=False, grid="full128")
    x = wl.normal_bf16((M, K), 1.0, seed=81)
    y = q8.q8_linear_w8a16_planes(x.to(DEV), q, s, _ws(M, N, K), out_dtype=torch.float32)
    torch.cuda.synchronize()
    rq, rs, _ = oracle.quantize_weight(W.numpy(), grid="full128")
    assert (rq == -128).any()
    y64, absum = oracle.linear_w8a16(wl.bf16_bits(x), rq, rs)
    _tight(y.cpu().numpy(), y64, absum, f"planes on the full grid M={M}")
