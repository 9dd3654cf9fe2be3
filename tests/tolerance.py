"""Output tolerances (the contract the CUDA path is held to against the oracle).

fp32 outputs: |y - y64| <= 1e-5 * sum_k |xhat_k s_w q_k| + 1e-6, with y64 the oracle's
fp64-accumulated value and the magnitude sum from the oracle too.

bf16 outputs: within 2 bf16 ulps of the oracle's fp64 value rounded once to bf16, or --
near cancellation, where |y| is far below the magnitude sum -- within the fp32 bound above
plus half a bf16 ulp (the final rounding).  Returns how many elements needed the second
clause so that tests can report it.
"""
import numpy as np

import oracle


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 2.0 ** -126)))
    return 2.0 ** (np.maximum(e, -126) - 7)


def check_f32(y: np.ndarray, y64: np.ndarray, absum: np.ndarray, what: str = "") -> None:
    y = np.asarray(y, np.float64)
    err = np.abs(y - y64)
    bound = 1e-5 * absum + 1e-6
    bad = ~(err <= bound)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} fp32 outputs out of tolerance; first at "
                             f"{tuple(i)}: got {y[tuple(i)]!r}, oracle {y64[tuple(i)]!r}, "
                             f"bound {bound[tuple(i)]!r}")


def check_bf16(y_bits: np.ndarray, y64: np.ndarray, absum: np.ndarray, what: str = "") -> int:
    y = bf16_bits_to_f32(y_bits).astype(np.float64)
    ref = bf16_bits_to_f32(oracle.round_bf16(y64)).astype(np.float64)
    ulp = bf16_ulp(ref)
    ok_ulp = np.abs(y - ref) <= 2 * ulp
    ok_abs = np.abs(y - y64) <= 1e-5 * absum + 1e-6 + 0.5 * ulp
    bad = ~(ok_ulp | ok_abs)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} bf16 outputs out of tolerance; first at {i}: "
                             f"got {y[i]!r}, oracle {y64[i]!r} (bf16 {ref[i]!r})")
    return int((~ok_ulp & ok_abs).sum())
