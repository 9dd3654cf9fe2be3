"""W8A8 linear outputs as exact functions of the int32 accumulators.

The W8A8 epilogue is y = s_w * (s1 * (acc1 - z1 * wsum) + s2 * (acc2 - z2 * wsum))
([SmolVLM-Q8] Q8Linear.forward, the delegated linear_q8ta_q8csw with its weight_sums
operand).  The float tolerance of the other W8A8 tests admits tens of accumulator units at
K = 4096, so an accumulation bug of a few units would pass there.  Here every float step
is made exact instead:

  * s_w = 1 and s1, s2 are powers of two, so each scale multiply is exact;
  * the activations are built on the quantization grid, x = (c - z1) * s1 (+ e * s2 for
    the second pass), so the static quantizer returns the chosen codes c (and e + z2)
    without rounding, with z1 and z2 nonzero so that the zero-point terms are exercised;
  * t = acc - z * wsum stays below 2^24 in magnitude (asserted), so its fp32 conversion
    is exact, and for two passes s1 * t1 + s2 * t2 is itself an fp32 number (asserted).

Then y must equal, bit for bit, the value formed from the oracle's exact integer
accumulators, and a single wrong accumulator unit changes y by at least s2.  The cases
cover the GEMV (M <= 16) and the tensor-core GEMM (M > 16) with both its one-pass tile
widths (256 and 128 weight rows) and the two-pass form."""
import numpy as np
import pytest
import torch

import int8_quantized_linear_q8_b200 as q8
import oracle
from int8_quantized_linear_q8_b200 import build as q8build

pytestmark = pytest.mark.gpu
DEV = "cuda"

S1 = 2.0 ** -3            # first-pass scale (power of two)
Z1 = -37                  # first-pass zero point (nonzero)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q8build.build()
    q8.lib()
    yield
    assert q8.q8_last_device_status() == q8.Q8_OK


def _weights(N, K, seed):
    """Any int8 codes (both grids' ranges, -128 included), unit scales, their code sums."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randint(-128, 128, (N, K), dtype=torch.int8, generator=g)
    wsum = q.to(torch.int64).sum(1).to(torch.int32)
    return q, torch.ones(N, dtype=torch.float32), wsum


def _x_one_pass(M, K, seed):
    """x on the first-pass grid: codes over the whole int8 range, plus about 1% of values
    far outside it (the quantizer clamps them to -128 / 127)."""
    g = torch.Generator().manual_seed(seed)
    c = torch.randint(-128, 128, (M, K), generator=g)
    v = (c - Z1).to(torch.float32)
    far = torch.rand(M, K, generator=g) < 0.01
    v = torch.where(far, torch.sign(v + 0.5) * 1000.0, v)
    return v * S1                                    # exact: small integers times 2^-3


def _x_two_pass_narrow(M, K, seed, z2):
    """First-pass codes within 1 of z1 (so t1 stays small) and a residual of e * s2 with
    s2 = s1 / 256: the second-pass codes are e + z2.  |e| < 128 keeps e * s2 below half a
    first-pass step (no rounding tie), and e + z2 stays inside [-128, 127]."""
    g = torch.Generator().manual_seed(seed)
    c = torch.randint(-1, 2, (M, K), generator=g)
    e = torch.randint(max(-127, -128 - z2), min(128, 128 - z2), (M, K), generator=g)
    return (c * 256 + e).to(torch.float32) * (S1 / 256.0)


def _x_two_pass_wide(M, K, seed):
    """s2 = s1: values v * s1 with v up to +-300, so the first pass clamps many of them and
    the second pass encodes what the first one clipped (wide codes in both passes)."""
    g = torch.Generator().manual_seed(seed)
    v = torch.randint(-300, 301, (M, K), generator=g)
    return v.to(torch.float32) * S1


def _run(x, q, s_w, wsum, first, second, rows):
    y = q8.q8_linear_w8a8(x.to(DEV), first, q.to(DEV), wsum.to(DEV), s_w.to(DEV), second=second)
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    y64, _, acc1, acc2 = oracle.linear_w8a8(x.numpy(), first, q.numpy(), s_w.numpy(),
                                           second=second, rows=rows)
    ws = wsum.numpy().astype(np.int64)[None, :]
    t1 = acc1.astype(np.int64) - first[1] * ws
    assert np.abs(t1).max() < 2 ** 24, "test inputs must keep acc1 - z1 wsum exact in fp32"
    if second is None:
        units, unit = t1, first[0]
    else:
        t2 = acc2.astype(np.int64) - second[1] * ws
        assert np.abs(t2).max() < 2 ** 24, "test inputs must keep acc2 - z2 wsum exact in fp32"
        ratio = int(round(first[0] / second[0]))
        assert ratio * second[0] == first[0]
        units, unit = ratio * t1 + t2, second[0]
    assert np.abs(units).max() < 2 ** 24, "the exact output must be an fp32 number"
    want = (units.astype(np.float64) * unit).astype(np.float32)      # exact conversion
    assert np.array_equal(want.astype(np.float64), units * float(unit))
    assert np.array_equal(y64.astype(np.float32), want)              # the oracle agrees
    got = y if rows is None else y[rows]
    bad = got.view(np.uint32) != want.view(np.uint32)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{bad.sum()} outputs differ from the exact accumulator value; "
                             f"first at {i}: got {got[i]!r} = {got[i] / unit!r} units, "
                             f"exact {want[i]!r} = {units[i]} units")
    return units


# M <= 16 and small problems (under 6 MB of 16-row weight passes: 32 x 960 x 960,
# 64 x 960 x 960, 40 x 300 x 512) run the GEMV, larger ones the tensor-core GEMM.  One pass:
# 256-row weight tiles where they give at least two tiles per SM (4096 x 4096), 128-row
# tiles otherwise.
ONE_PASS = [(1, 2560, 960), (5, 960, 960), (16, 1000, 4096), (17, 300, 4096),
            (32, 960, 960), (40, 300, 512),
            (256, 960, 960), (2048, 2560, 960), (300, 520, 4096), (4096, 4096, 4096)]


@pytest.mark.parametrize("M,N,K", ONE_PASS)
def test_w8a8_one_pass_exact_accumulators(M, N, K):
    q, s_w, wsum = _weights(N, K, seed=7000 + N + K)
    x = _x_one_pass(M, K, seed=7100 + M)
    rows = None if M <= 300 else [0, 1, 127, 128, 129, M // 2, M - 1]
    _run(x, q, s_w, wsum, (S1, Z1), None, rows)


TWO_PASS = [(1, 2560, 960), (5, 960, 960), (16, 1000, 4096), (64, 960, 960), (256, 2560, 960),
            (2048, 960, 960), (300, 520, 4096), (2048, 4096, 4096)]


@pytest.mark.parametrize("M,N,K", TWO_PASS)
def test_w8a8_two_pass_exact_accumulators_narrow(M, N, K):
    """s2 = s1 / 256, z2 = 3: y / s2 = 256 t1 + t2 separates the two accumulators."""
    z2 = 3
    q, s_w, wsum = _weights(N, K, seed=7200 + N + K)
    x = _x_two_pass_narrow(M, K, seed=7300 + M, z2=z2)
    rows = None if M <= 300 else [0, 1, 127, 128, 129, M // 2, M - 1]
    _run(x, q, s_w, wsum, (S1, Z1), (S1 / 256.0, z2), rows)


@pytest.mark.parametrize("M,N,K", [(4, 2560, 960), (16, 1000, 4096), (256, 960, 960),
                                   (2048, 4096, 4096)])
def test_w8a8_two_pass_exact_accumulators_wide(M, N, K):
    """s2 = s1, z2 = -5: wide codes in both passes, y / s1 = t1 + t2."""
    q, s_w, wsum = _weights(N, K, seed=7400 + N + K)
    x = _x_two_pass_wide(M, K, seed=7500 + M)
    rows = None if M <= 300 else [0, 1, 127, 128, 129, M // 2, M - 1]
    _run(x, q, s_w, wsum, (S1, Z1), (S1, -5), rows)
