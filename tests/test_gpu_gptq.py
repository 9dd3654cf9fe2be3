"""GPU parity of the offline GPTQ path against the oracle: the calibration Hessian
(hessians, SmolVLM q8 page) and gptq_int8 (same page) are computed in float64 with every sum
in ascending order on both sides, so Hessian entries, codes, scales and code sums must be
the same bits."""
import numpy as np
import pytest
import torch

import int8_quantized_linear_q8_b200 as q8
import oracle
import q8_workloads as wl
from int8_quantized_linear_q8_b200 import build as q8build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q8build.build()
    q8.lib()
    yield
    assert q8.q8_last_device_status() == q8.Q8_OK


def _calib_x(R, K, seed, dead=()):
    """Correlated calibration inputs (mixed Gaussian columns); `dead` columns never active."""
    g = torch.Generator().manual_seed(seed)
    z = torch.randn(R, K, generator=g, dtype=torch.float64)
    mix = torch.eye(K, dtype=torch.float64) + \
        0.6 * torch.randn(K, K, generator=g, dtype=torch.float64) / K ** 0.5
    x = (z @ mix).float()
    for k in dead:
        x[:, k] = 0.0
    return x


@pytest.mark.parametrize("K,batches", [(64, [100]), (208, [1000, 37, 300]), (960, [33, 512])])
def test_hessian_accumulate_bit_exact(K, batches):
    xs = [_calib_x(r, K, seed=800 + i + K, dead=(3,)) for i, r in enumerate(batches)]
    H = None
    for i, x in enumerate(xs):
        H = q8.q8_hessian_accumulate(x.to(DEV), H, reset=(i == 0))
    ref = oracle.hessian([x.numpy() for x in xs])
    assert np.array_equal(H.cpu().numpy(), ref)


def _gptq_case(N, K, block, R, dead, seed):
    x = _calib_x(R, K, seed=seed, dead=dead)
    H = q8.q8_hessian_accumulate(x.to(DEV))
    W = wl.weight(N, K, seed=seed + 1)
    if dead:
        W[:, dead[0]] = 0.05                          # a dead column with weight in it
    q, s, ws = q8.q8_gptq_int8(W.to(DEV), H, block=block)
    torch.cuda.synchronize()
    return W, H.cpu().numpy(), q, s, ws


@pytest.mark.parametrize("N,K,block,R,dead", [
    (300, 512, 128, 2000, (7, 300)),        # the page's block size, dead columns
    (37, 208, 100, 500, ()),                # ragged last block (208 = 2 * 100 + 8)
    (64, 256, 1, 300, (0,)),                # one column per block
    (17, 512, 256, 200, (511,)),            # R < K: positive definite only after damping
])
def test_gptq_bit_exact(N, K, block, R, dead):
    W, H, q, s, ws = _gptq_case(N, K, block, R, dead, seed=810 + K)
    rq, rs, rws = oracle.gptq_int8(W.numpy(), H, block=block)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(ws.cpu().numpy(), rws)
    if dead:
        assert not rq[:, list(dead)].any()


def test_gptq_llama_shape_sampled():
    """N = 11008, K = 4096 (a Llama MLP up-projection) with 1024 calibration rows: Hessian
    rows sampled against the oracle's Gram rows, codes of sampled weight rows against the
    oracle (which needs the whole inverse-Hessian factor, but only those rows of W)."""
    N, K, R = 11008, 4096, 1024
    x = _calib_x(R, K, seed=830, dead=(11,))
    H = q8.q8_hessian_accumulate(x.to(DEV))
    hrows = [0, 11, 2047, 4095]
    assert np.array_equal(H.cpu().numpy()[hrows], oracle.gram(x.numpy(), rows=hrows))
    W = wl.weight(N, K, seed=831)
    q, s, ws = q8.q8_gptq_int8(W.to(DEV), H)
    torch.cuda.synchronize()
    rows = [0, 1, 5000, 11007]
    rq, rs, rws = oracle.gptq_int8(W.numpy(), H.cpu().numpy(), rows=rows)
    assert np.array_equal(q.cpu().numpy()[rows], rq)
    assert np.array_equal(s.cpu().numpy()[rows].view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(ws.cpu().numpy()[rows], rws)


def test_gptq_not_positive_definite_reports():
    """A Hessian with a negative diagonal stays indefinite after damping: the call records a
    device failure instead of faulting, and the status word is cleared by reading it."""
    K, N = 64, 8
    H = -torch.eye(K, dtype=torch.float64, device=DEV)
    W = wl.weight(N, K, seed=840).to(DEV)
    q8.q8_gptq_int8(W, H)
    assert q8.q8_last_device_status() == q8.Q8_ERR_DEVICE
    assert q8.q8_last_device_status() == q8.Q8_OK


def test_gptq_codes_feed_the_linears():
    """GPTQ codes and scales are operands of q8_linear_w8a16 like any weight_int8 codes."""
    N, K, M = 256, 512, 4
    W, H, q, s, _ = _gptq_case(N, K, 128, 1500, (), seed=850)
    x = wl.normal_bf16((M, K), 1.0, seed=851)
    y = q8.q8_linear_w8a16(x.to(DEV), q, s, out_dtype=torch.float32)
    torch.cuda.synchronize()
    y64, absum = oracle.linear_w8a16(wl.bf16_bits(x), q.cpu().numpy(), s.cpu().numpy())
    from tolerance import check_f32
    check_f32(y.cpu().numpy(), y64, absum, "w8a16 on GPTQ codes")
