"""The fp32 steps of the int8 8da4w GEMM's epilogue, checked exactly on the host.

Per element and group that epilogue receives t = 16 * sum_{k in g} xq * q4 (int32, from
the MMA on 16 * q4) and computes, in fp32:
    f = float with the bits of (t + bits(1.5 * 2^23))        (= 1.5 * 2^23 + t)
    c = fma(z, 16 * Q_g, 1.5 * 2^23)
    acc = fma(gs / 16, f - c, acc)
The bf16 GEMM computes acc = fma(gs, T_g, acc) with T_g = sum (xq - z) q4 exact in fp32.
Both must give the same fp32 bits (the GPU tests compare the two paths and the oracle);
here every step is evaluated with exact rationals over the full operand ranges, the
extreme partial sums |t| = 2^22 (G = 256, all codes -128 and -8) included."""
from fractions import Fraction

import numpy as np

MAGIC_F = 12582912.0
MAGIC_I = 0x4B400000


def f32(x):
    """Round a rational to the nearest fp32, ties to the even significand."""
    v = np.float32(float(x))             # within one fp32 step of the answer
    cands = [np.nextafter(v, np.float32(-np.inf)), v, np.nextafter(v, np.float32(np.inf))]
    dist = [abs(Fraction(float(c)) - x) for c in cands]
    best = min(dist)
    ties = [c for c, d in zip(cands, dist) if d == best]
    even = [c for c in ties if int(np.float32(c).view(np.uint32)) % 2 == 0]
    return (even or ties)[0]


def fma32(a, b, c):
    return f32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def bits_to_f32(i):
    return np.array([i], dtype=np.int64).astype(np.uint32).view(np.float32)[0]


def epilogue_i8(t, z, q16, gs, acc):
    f = bits_to_f32(int(t) + MAGIC_I)
    assert Fraction(float(f)) == MAGIC_F + t                        # exact conversion
    c = fma32(np.float32(z), np.float32(q16), np.float32(MAGIC_F))
    assert Fraction(float(c)) == MAGIC_F + z * q16                  # exact zero-point term
    d = f32(Fraction(float(f)) - Fraction(float(c)))
    assert Fraction(float(d)) == t - z * q16                        # exact 16 * T_g
    return fma32(np.float32(gs) * np.float32(0.0625), d, acc)


def epilogue_bf16(T, gs, acc):
    return fma32(np.float32(gs), np.float32(T), acc)


def test_i8_epilogue_matches_bf16_epilogue():
    rng = np.random.default_rng(2024)
    cases = []
    for G in (32, 64, 128, 256):
        # extremes: every product at its largest magnitude, both signs
        for xq, q in ((-128, -8), (-128, 7), (127, -8), (127, 7)):
            for z in (-128, 0, 127):
                cases.append((16 * xq * q * G, z, 16 * q * G))
        for _ in range(300):
            xq = rng.integers(-128, 128, G)
            q = rng.integers(-8, 8, G)
            z = int(rng.integers(-128, 128))
            cases.append((int(16 * (xq * q).sum()), z, int(16 * q.sum())))
    for t, z, q16 in cases:
        assert abs(t) <= 2 ** 22
        T = Fraction(t - z * q16, 16)
        assert T.denominator == 1 and abs(T) < 2 ** 24
        gs = np.float32(rng.uniform(1e-4, 1.0))
        acc = np.float32(rng.normal() * 10)
        a = epilogue_i8(t, z, q16, gs, acc)
        b = epilogue_bf16(T, gs, acc)
        assert np.float32(a).view(np.uint32) == np.float32(b).view(np.uint32), (t, z, q16)


def test_magic_conversion_bounds():
    """The bit trick holds exactly on [-2^22, 2^22] (the ends land on 2^23 and 2^24)."""
    for t in (-2 ** 22, -2 ** 22 + 1, -1, 0, 1, 2 ** 22 - 1, 2 ** 22):
        assert Fraction(float(bits_to_f32(t + MAGIC_I))) == MAGIC_F + t
