"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the quantized linear: it only draws random
numbers (torch CPU generators, fixed seeds) in the shapes, distributions and
structure of the workloads the source pages quantize, and names the workload
configurations.  Both the CUDA path and the CPU oracle are fed from here.

bf16 tensors are produced by rounding an fp32 draw to bf16 (torch's cast) and
are handed to the oracle as their uint16 bit patterns.
"""
from __future__ import annotations

import dataclasses
from typing import List, Tuple

import numpy as np
import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, seed: int) -> torch.Tensor:
    """fp32 N(0, std^2) draw on the CPU."""
    return torch.randn(*shape, generator=_gen(seed), dtype=torch.float32) * float(std)


def normal_bf16(shape, std: float, seed: int) -> torch.Tensor:
    """bf16 tensor: an fp32 N(0, std^2) draw rounded to bf16."""
    return normal(shape, std, seed).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (the oracle's bf16 format)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def weight(N: int, K: int, seed: int, std: float = 0.02, zero_rows=()) -> torch.Tensor:
    """fp32 weight [N, K] ~ N(0, std^2), with the listed rows set to zero."""
    W = normal((N, K), std, seed)
    for r in zero_rows:
        W[r].zero_()
    return W


def outlier_columns(K: int, frac: float, seed: int) -> torch.Tensor:
    """max(1, round(frac*K)) distinct column indices, chosen by a seeded permutation."""
    n = max(1, int(round(frac * K)))
    return torch.randperm(K, generator=_gen(seed))[:n]


def activations_with_outliers(M: int, K: int, std: float, seed: int, cols: torch.Tensor,
                              factor: float = 50.0) -> torch.Tensor:
    """fp32 activations [M, K] ~ N(0, std^2) with the given columns scaled by `factor`
    (the 'massive activation' structure: a few channels far larger than the rest)."""
    x = normal((M, K), std, seed)
    x[:, cols] *= factor
    return x


# ----------------------------------------------------------------------------- configurations


@dataclasses.dataclass(frozen=True)
class Shape:
    K: int
    N: int


# (K, N) shapes of the W8A16 decode sweep and its activation rows M.
W8A16_SWEEP_SHAPES: List[Shape] = [Shape(960, 2560), Shape(2048, 8192), Shape(4096, 11008),
                                   Shape(4096, 32000)]
W8A16_SWEEP_M = (1, 4, 16)
W8A16_SWEEP_SEED_W = 1
W8A16_SWEEP_SEED_X = 2

# Single small parity case: one fp32 weight 256 x 512 with row 7 all zeros, M = 1.
PR1 = dict(N=256, K=512, zero_rows=(7,), seed=0, M=1)

# W8A8 static: K = 960, N in {960, 2560}, M in {1, 256, 2048}; x ~ N(0, 4^2) with 0.1% of
# the columns x50; per-tensor qparams from a 4096-row calibration draw.
W8A8_K = 960
W8A8_N = (960, 2560)
W8A8_M = (1, 256, 2048)
W8A8_X_STD = 4.0
W8A8_OUTLIER_FRAC = 0.001
W8A8_SEED_X = 3
W8A8_SEED_CALIB = 4
W8A8_SEED_W = 5
W8A8_SEED_COLS = 9
W8A8_CALIB_ROWS = 4096

# 8da4w: x bf16 N(0,1), K = 4096, N = 11008, M in {1, 64, 512, 4096}, G in {32, 128}.
Q4_K = 4096
Q4_N = 11008
Q4_M = (1, 64, 512, 4096)
Q4_G = (32, 128)
Q4_SEED_X = 6
Q4_SEED_W = 7

# Llama-shaped stack: 32 layers of (q, k, v, o: 4096x4096; gate, up: 4096->11008;
# down: 11008->4096); weights N(0, 0.02^2), seed 8 + layer.
LLAMA_LAYERS = 32
LLAMA_LINEARS: List[Tuple[str, int, int]] = [  # (name, K=in, N=out)
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 4096, 11008), ("up", 4096, 11008), ("down", 11008, 4096)]
LLAMA_PREFILL_M = 4096


def w8a8_inputs(M: int, K: int = W8A8_K, seed_x: int = W8A8_SEED_X):
    """(x [M,K], calibration draw [4096,K]) fp32 with the same outlier columns."""
    cols = outlier_columns(K, W8A8_OUTLIER_FRAC, W8A8_SEED_COLS)
    x = activations_with_outliers(M, K, W8A8_X_STD, seed_x, cols)
    calib = activations_with_outliers(W8A8_CALIB_ROWS, K, W8A8_X_STD, W8A8_SEED_CALIB, cols)
    return x, calib
