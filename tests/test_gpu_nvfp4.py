"""GPU parity of the NVFP4 weight-only twin (flashrt-structures schemes.py, W4A16Decode):
the quantizer's codes, E4M3 block scales and tensor scale bit for bit against the oracle,
and the W4A16 linear within the R11 / fp32 tolerances (the block-scaled weight is exact in
bf16, so only the accumulation order differs)."""
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


def _edge_weight(N, K, seed):
    W = wl.weight(N, K, seed=seed)
    W[0] = 0.0                                   # an all-zero row
    W[1, 16:48] = 0.0                            # zero blocks
    W[2, :16] *= 1e-7                            # blocks below the smallest E4M3 scale
    W[3, 5] = 0.6                                # the tensor's absmax (gsc from it)
    W[4, 32:48] = torch.tensor([0.25, -0.75, 1.25, -1.75, 2.5, -3.5, 5.0, 6.0,
                                0.0, -0.0, 3.0, -6.0, 0.5, 1.0, -1.5, 2.0]) * 0.01
    return W


@pytest.mark.parametrize("N,K", [(256, 512), (2560, 960), (37, 96), (11008, 4096),
                                 (32000, 4096)])
def test_quantize_weight_nvfp4_bit_exact(N, K):
    W = _edge_weight(N, K, seed=5000 + K)
    q4, sf, gsc = q8.q8_quantize_weight_nvfp4(W.to(DEV))
    rq4, rsf, rg = oracle.quantize_weight_nvfp4(W.numpy())
    assert gsc.item() == float(rg) and np.float32(gsc.item()).view(np.uint32) == rg.view(np.uint32)
    assert np.array_equal(sf.cpu().numpy(), rsf)
    assert np.array_equal(q4.cpu().numpy(), rq4)


def test_quantize_weight_nvfp4_zero_tensor():
    W = torch.zeros(16, 64)
    q4, sf, gsc = q8.q8_quantize_weight_nvfp4(W.to(DEV))
    assert gsc.item() == 1.0 and not q4.any().item() and not sf.any().item()


def _w4_case(M, N, K, seed, out_dtype):
    W = _edge_weight(N, K, seed=seed) if N >= 5 else wl.weight(N, K, seed=seed)
    x = wl.normal_bf16((M, K), 1.0, seed=seed + 1)
    q4, sf, gsc = q8.q8_quantize_weight_nvfp4(W.to(DEV))
    y = q8.q8_linear_w4a16_nvfp4(x.to(DEV), q4, sf, gsc, out_dtype=out_dtype)
    torch.cuda.synchronize()
    rq4, rsf, rg = oracle.quantize_weight_nvfp4(W.numpy())
    return x, rq4, rsf, rg, y


@pytest.mark.parametrize("shape", wl.W8A16_SWEEP_SHAPES, ids=lambda s: f"K{s.K}xN{s.N}")
@pytest.mark.parametrize("M", wl.W8A16_SWEEP_M)
def test_w4a16_nvfp4_sweep_bf16(shape, M):
    """The W8A16 decode sweep's shapes with NVFP4 weights (sampled output rows at M = 16)."""
    x, rq4, rsf, rg, y = _w4_case(M, shape.N, shape.K, 5100 + shape.N % 977 + M, torch.bfloat16)
    y64, absum = oracle.linear_w4a16_nvfp4(wl.bf16_bits(x), rq4, rsf, rg)
    check_bf16(_bits(y), y64, absum, f"w4a16 sweep M={M} {shape}")


@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (3, 33, 96), (8, 1000, 960), (9, 129, 2048),
                                   (16, 300, 11008), (20, 77, 160), (40, 64, 4096)])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_w4a16_nvfp4_ragged(M, N, K, out):
    x, rq4, rsf, rg, y = _w4_case(M, N, K, 5200 + M + N, out)
    y64, absum = oracle.linear_w4a16_nvfp4(wl.bf16_bits(x), rq4, rsf, rg)
    if out == torch.float32:
        check_f32(y.cpu().numpy(), y64, absum, "w4a16 ragged fp32")
    else:
        check_bf16(_bits(y), y64, absum, "w4a16 ragged bf16")


def test_w4a16_nvfp4_codes_of_every_value():
    """Weights made of all 16 codes with a spread of block scales (built by hand, not by
    the quantizer): the kernel's E2M1 / E4M3 decoding, sign handling included, against the
    oracle."""
    N, K, M = 64, 512, 4
    g = torch.Generator().manual_seed(5300)
    q4 = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, generator=g)
    sf = torch.randint(0, 127, (N, K // 16), dtype=torch.uint8, generator=g)   # no NaN byte
    gsc = torch.tensor([0.75])
    x = wl.normal_bf16((M, K), 1.0, seed=5301)
    y = q8.q8_linear_w4a16_nvfp4(x.to(DEV), q4.to(DEV), sf.to(DEV), gsc.to(DEV),
                                 out_dtype=torch.float32)
    y64, absum = oracle.linear_w4a16_nvfp4(wl.bf16_bits(x), q4.numpy(), sf.numpy(), 0.75)
    check_f32(y.cpu().numpy(), y64, absum, "w4a16 all codes")


def test_w4a16_nvfp4_empty_m():
    q4 = torch.zeros(16, 32, dtype=torch.uint8, device=DEV)
    sf = torch.zeros(16, 4, dtype=torch.uint8, device=DEV)
    gsc = torch.ones(1, device=DEV)
    y = q8.q8_linear_w4a16_nvfp4(torch.zeros(0, 64, dtype=torch.bfloat16, device=DEV), q4, sf, gsc)
    assert y.shape == (0, 16)
