"""The allocation-free W8A8 entry point (q8_linear_w8a8_noalloc), for callers that cannot
allocate device memory (a runtime that owns all device memory, a loop that cannot afford
cudaMalloc's synchronisation, a bare C caller with no allocator).  It must compute what
q8_linear_w8a8 computes with a caller workspace.  This file is collected last."""
import ctypes

import numpy as np
import pytest
import torch

import int8_quantized_linear_q8_b200 as q8
import oracle
import q8_workloads as wl
from int8_quantized_linear_q8_b200 import build as q8build
from tolerance import check_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q8build.build()
    q8.lib()


def _case(M, N, K, seed):
    x = wl.normal((M, K), 4.0, seed=seed)
    W = wl.weight(N, K, seed=seed + 1)
    mm = torch.empty(2, device=DEV)
    q8.q8_observe_minmax(x.to(DEV), mm, reset=True)
    first = q8.q8_qparams_from_minmax(*mm.cpu().tolist())
    second = (float(np.float32(first[0]) / np.float32(255.0)), 0)
    q, s, ws = q8.q8_quantize_weight(W.to(DEV))
    return x, W, first, second, q, s, ws


@pytest.mark.parametrize("M,N,K", [(4, 2560, 960), (512, 1000, 4096)])
@pytest.mark.parametrize("two", [False, True])
def test_noalloc_matches_workspace_entry_point(M, N, K, two):
    """Two calls in a row on different inputs, each against q8_linear_w8a8 with a workspace
    (same tolerance as the parity tests, measured against the oracle's magnitude sums)."""
    for call, seed in enumerate((700 + M, 800 + M)):
        x, W, first, second, q, s, ws = _case(M, N, K, seed)
        sec = second if two else None
        xd = x.to(DEV)
        y_ref = q8.q8_linear_w8a8(xd, first, q, ws, s, second=sec)
        y_new = torch.empty(M, N, device=DEV)
        q8.q8_linear_w8a8_noalloc(xd, first, q, ws, s, second=sec, y=y_new)
        torch.cuda.synchronize()
        rq, rs, _ = oracle.quantize_weight(W.numpy())
        rows = None if M <= 64 else [0, 1, M // 2, M - 1]
        y64, absum, _, _ = oracle.linear_w8a8(x.numpy(), first, rq, rs, second=sec, rows=rows)
        got_new = y_new.cpu().numpy() if rows is None else y_new.cpu().numpy()[rows]
        got_ref = y_ref.cpu().numpy() if rows is None else y_ref.cpu().numpy()[rows]
        check_f32(got_new, got_ref.astype(np.float64), absum, f"no-alloc vs workspace, call {call}")
        check_f32(got_new, y64, absum, f"no-alloc vs oracle, call {call}")
    assert q8.q8_last_device_status() == q8.Q8_OK


def test_noalloc_rejects_oversize():
    """Beyond the built-in 16 MiB the call fails with Q8_ERR_WORKSPACE and writes nothing."""
    M, K, N = 4096, 4096, 16
    x = torch.zeros(M, K, device=DEV)
    q = torch.zeros(N, K, dtype=torch.int8, device=DEV)
    ws = torch.zeros(N, dtype=torch.int32, device=DEV)
    s = torch.ones(N, device=DEV)
    y = torch.full((M, N), 7.0, device=DEV)
    assert q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, M, N, K, 1) > q8.Q8_NOALLOC_SCRATCH_BYTES
    with pytest.raises(q8.Q8Error) as e:
        q8.q8_linear_w8a8_noalloc(x, (0.1, 0), q, ws, s, second=(0.1 / 255, 0), y=y)
    assert e.value.status == q8.Q8_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (y == 7.0).all()
