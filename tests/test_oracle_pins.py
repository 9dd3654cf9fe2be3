"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

Nothing here compares the oracle with itself.  Each check is one of:
  * a hand-worked value from tests/golden/ (each file cites the page rule it follows);
  * brute force in exact rational arithmetic (tests/exact.py) on tiny inputs;
  * a closed-form bound or invariant (nearest-grid error, two-pass bound, zero point);
  * a special case that reduces to a library routine (numpy matmul, torch bf16 cast).
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import q8_workloads as wl
from exact import bf16_bits_to_fraction, f32, rn32, rn_bf16, rne_int

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([part.split() for part in line.split("|")])
    return rows


def _bf16(values):
    return wl.bf16_bits(torch.tensor(values, dtype=torch.float32).to(torch.bfloat16))


# ----------------------------------------------------------------- golden rows


def test_golden_weight_rows():
    """Int8Linear's quantize_weight rule (ROCm INT8 page) on hand-worked rows."""
    rows = _parse("weight_int8_rows.txt")
    W = np.array([[float(v) for v in r[0]] for r in rows], np.float32)
    q, s, ws = oracle.quantize_weight(W)
    for i, r in enumerate(rows):
        assert q[i].tolist() == [int(v) for v in r[2]], f"row {i} codes"
        assert ws[i] == int(r[3][0]), f"row {i} code sum"
        assert s[i] == pytest.approx(float(r[1][0]), rel=1e-7), f"row {i} scale"
    assert s[0] == 1.0 and s[1] == 2.0 and s[2] == 1.0      # exact scales


def test_golden_activation_rows():
    """choose_qparams_affine (executorch PR #21229) on hand-worked rows."""
    rows = _parse("act_qparams_rows.txt")
    x = _bf16([[float(v) for v in r[0]] for r in rows])
    s, z, xq = oracle.choose_qparams(x)
    for i, r in enumerate(rows):
        assert z[i] == int(r[1][0]), f"row {i} zero point"
        assert xq[i].tolist() == [int(v) for v in r[2]], f"row {i} codes"
    assert s[0] == np.float32(4.0) / np.float32(255.0)
    assert s[1] == np.finfo(np.float32).eps
    assert s[2] == np.float32(4.0) / np.float32(255.0)


def test_golden_q4_groups():
    """int4 group-symmetric codes and nibble packing on hand-worked groups."""
    rows = _parse("weight_q4gs_groups.txt")
    W = np.array([[float(v) for r in rows for v in r[0]]], np.float32)   # 1 x 12, G = 4
    q4, gs = oracle.quantize_weight_q4gs(W, 4)
    want_bytes = [int(b, 16) for r in rows for b in r[3]]
    assert q4[0].tolist() == want_bytes
    assert gs[0].tolist() == [float(r[1][0]) for r in rows]


def test_golden_q4gs_zero_fold():
    """The 8da4w zero-point fold c[n] (row sum of the dequantized weight) on hand-worked
    rows, including a zero group, a negative sum and the final fp32 rounding."""
    rows = _parse("q4gs_zero_fold_rows.txt")
    W = np.array([[float(v) for v in r[0]] for r in rows], np.float32)
    q4, gs = oracle.quantize_weight_q4gs(W, 4)
    c = oracle.q4gs_zero_fold(q4, gs, 4)
    for i, r in enumerate(rows):
        assert Fraction(float(c[i])) == Fraction(r[1][0]), f"row {i}"


def test_q4gs_zero_fold_exact_row_sums():
    """c[n] is the nearest fp32 to the exact rational row sum of gs * code (codes decoded
    here from the packed bytes), for random weights, both group sizes and zero groups."""
    W = wl.weight(24, 512, seed=35).numpy()
    W[3, 64:192] = 0.0
    W[5] *= 1e-20
    for G in (32, 128):
        q4, gs = oracle.quantize_weight_q4gs(W, G)
        c = oracle.q4gs_zero_fold(q4, gs, G)
        for n in range(W.shape[0]):
            exact = Fraction(0)
            for g in range(512 // G):
                S = 0
                for k in range(g * G, (g + 1) * G):
                    b = int(q4[n, k // 2])
                    nib = (b >> 4) if k & 1 else (b & 0xF)
                    S += nib - 16 if nib >= 8 else nib
                exact += Fraction(float(gs[n, g])) * S
            assert Fraction(float(c[n])) == rn32(exact), f"G={G} row {n}"


# ------------------------------------------------------ weight codes, brute force


def _weight_codes_exact(w_row):
    amax = max(abs(f32(v)) for v in w_row)
    s = rn32(amax / 127) if amax else Fraction(0)
    if s == 0:
        return Fraction(1), [0] * len(w_row)
    codes = [max(-127, min(127, rne_int(rn32(f32(v) / s)))) for v in w_row]
    return s, codes


def test_quantize_weight_exact_rational():
    W = wl.weight(12, 37, seed=11).numpy()
    W[3] = 0.0
    W[5, :] = 0.0
    W[5, 7] = -1e-3
    W[8] *= 1e-30                                    # tiny but normal scales
    q, s, ws = oracle.quantize_weight(W)
    for n in range(W.shape[0]):
        s_ex, codes = _weight_codes_exact(W[n])
        assert Fraction(float(s[n])) == s_ex
        assert q[n].tolist() == codes
        assert int(ws[n]) == sum(codes)


def _find_div_vs_recip_case():
    """A weight row where round(w / s) and round(w * (1/s)) differ in fp32."""
    rng = np.random.default_rng(5)
    for _ in range(200000):
        amax = np.float32(rng.uniform(0.5, 2.0))
        s = amax / np.float32(127.0)
        k = int(rng.integers(-120, 120))
        w = np.float32((k + 0.5) * float(s))
        if abs(w) >= amax:
            continue
        by_div = rne_int(rn32(f32(w) / f32(s)))
        by_rec = rne_int(rn32(f32(w) * rn32(1 / f32(s))))
        if by_div != by_rec:
            return np.array([[amax, w]], np.float32), by_div
    raise AssertionError("no case found")


def test_weight_codes_divide_not_reciprocal():
    """The ROCm page divides (round(w / scale)); a case where a reciprocal would differ."""
    W, want = _find_div_vs_recip_case()
    q, _, _ = oracle.quantize_weight(W)
    assert int(q[0, 1]) == want


def test_weight_codes_nearest_grid_point():
    """|q*s - w| <= s/2 (up to the fp32 division) and ties go to the even code."""
    W = wl.weight(64, 256, seed=12).numpy()
    q, s, _ = oracle.quantize_weight(W)
    err = np.abs(q.astype(np.float64) * s[:, None].astype(np.float64) - W.astype(np.float64))
    assert np.all(err <= s[:, None] * (0.5 + 2.0 ** -20))
    assert np.abs(q).max() == 127                   # the absmax element of each row hits 127
    assert np.all(np.abs(q).max(axis=1) == 127)


def test_zero_row_rule_and_clamp():
    """All-zero row: scale 1.0, codes 0 (ROCm page); p3's 'scale 0' reading is not used."""
    W = np.zeros((3, 16), np.float32)
    W[1, 4] = 3.0
    q, s, ws = oracle.quantize_weight(W)
    assert s[0] == 1.0 and s[2] == 1.0 and not q[0].any() and not q[2].any()
    assert q[1, 4] == 127 and ws[1] == 127


# -------------------------------------------------------- activation codes


def _act_codes_exact(x_vals, s, z):
    inv = rn32(1 / s)
    out = []
    for v in x_vals:
        t = rne_int(rn32(v * inv)) + z
        out.append(max(-128, min(127, t)))
    return out


def _qparams_exact(mn, mx):
    mn = min(mn, Fraction(0))
    mx = max(mx, Fraction(0))
    s = rn32(rn32(mx - mn) / 255)
    eps = Fraction(2) ** -23
    if s < eps:
        s = eps
    z = max(-128, min(127, -128 - rne_int(rn32(mn / s))))
    return s, z


def test_choose_qparams_exact_rational():
    xt = wl.normal_bf16((9, 33), 1.0, seed=13)
    xt[2] = torch.abs(xt[2])                         # positive-only row
    xt[3] = -torch.abs(xt[3])                        # negative-only row
    xt[4] = 0.0                                      # all zero
    xt[5] *= 1000.0
    bits = wl.bf16_bits(xt)
    s, z, xq = oracle.choose_qparams(bits)
    for m in range(bits.shape[0]):
        vals = [bf16_bits_to_fraction(b) for b in bits[m]]
        s_ex, z_ex = _qparams_exact(min(vals), max(vals))
        assert Fraction(float(s[m])) == s_ex, m
        assert int(z[m]) == z_ex, m
        assert xq[m].tolist() == _act_codes_exact(vals, s_ex, z_ex), m


def test_activation_code_invariants():
    """Real 0 maps to z; the row min maps to -128 and the max to 127 when the row
    straddles 0 (the affine grid's end points)."""
    bits = wl.bf16_bits(wl.normal_bf16((64, 128), 1.0, seed=14))
    s, z, xq = oracle.choose_qparams(bits)
    vals = bits.view(np.uint16).astype(np.uint32) << 16
    xf = vals.view(np.float32).reshape(bits.shape)
    for m in range(xf.shape[0]):
        assert xq[m, np.argmin(xf[m])] == -128
        assert xq[m, np.argmax(xf[m])] == 127
    zero_bits = _bf16([[0.0, 1.0, -2.0]])
    s0, z0, xq0 = oracle.choose_qparams(zero_bits)
    assert xq0[0, 0] == z0[0]


def test_qparams_from_minmax_matches_row_rule():
    """The per-tensor observer formula and the per-row one are the same function."""
    bits = wl.bf16_bits(wl.normal_bf16((4, 50), 2.0, seed=15))
    s, z, _ = oracle.choose_qparams(bits, want_codes=False)
    xf = (bits.astype(np.uint32) << 16).view(np.float32)
    for m in range(4):
        s_t, z_t = oracle.qparams_from_minmax(xf[m].min(), xf[m].max())
        assert (np.float32(s_t), z_t) == (s[m], z[m])
    s_ex, z_ex = _qparams_exact(Fraction(-1), Fraction(3))
    assert oracle.qparams_from_minmax(-1.0, 3.0) == (float(s_ex), z_ex)
    # ranges that exclude 0 are widened to contain it (golden activation row 2 by hand)
    s425 = float(np.float32(4.0) / np.float32(255.0))
    assert oracle.qparams_from_minmax(1.0, 4.0) == (s425, -128)
    assert oracle.qparams_from_minmax(-4.0, -1.0) == (s425, 127)


def test_static_codes_use_fp32_reciprocal():
    """fake_quant (SmolVLM q8 page) multiplies by 1/s; exact-rational check of codes and of
    the residual r = x - (xq1 - z1) * s1, each step rounded to fp32."""
    x = wl.normal((5, 40), 4.0, seed=16).numpy()
    s1, z1 = oracle.qparams_from_minmax(-9.0, 11.0)
    s2, z2 = float(np.float32(s1) / np.float32(255.0)), 0
    xq1, xq2 = oracle.static_quant(x, (s1, z1), (s2, z2))
    S1, S2 = f32(s1), f32(s2)
    for m in range(x.shape[0]):
        vals = [f32(v) for v in x[m]]
        c1 = _act_codes_exact(vals, S1, z1)
        assert xq1[m].tolist() == c1
        r = [rn32(v - rn32((c - z1) * S1)) for v, c in zip(vals, c1)]
        assert xq2[m].tolist() == _act_codes_exact(r, S2, z2)


def _find_recip_vs_div_act_case():
    """An activation x and scale s where round(x * (1/s)) and round(x / s) differ in fp32."""
    rng = np.random.default_rng(7)
    for _ in range(200000):
        s = np.float32(rng.uniform(0.01, 0.1))
        k = int(rng.integers(-100, 100))
        x = np.float32((k + 0.5) * float(s))
        by_rec = rne_int(rn32(f32(x) * rn32(1 / f32(s))))
        by_div = rne_int(rn32(f32(x) / f32(s)))
        if by_rec != by_div:
            return x, s, by_rec
    raise AssertionError("no case found")


def test_activation_codes_multiply_by_reciprocal():
    """fake_quant / quantize_per_tensor multiply by 1/s; a case where dividing would differ."""
    x, s, want = _find_recip_vs_div_act_case()
    xq1, _ = oracle.static_quant(np.array([[x]], np.float32), (float(s), 0))
    assert int(xq1[0, 0]) == max(-128, min(127, want))


def test_quant_error_bounds_single_and_two_pass():
    """Single pass: |x - dq(q(x))| <= s1/2.  Two passes with s2 = s1/255, z2 = 0:
    |x - dq1 - dq2| <= s1/510 (SmolVLM q8 page, module docstring), up to fp32 rounding."""
    s1, z1 = oracle.qparams_from_minmax(-6.0, 6.0)
    lo, hi = (-128 - z1) * s1, (127 - z1) * s1
    x = np.random.default_rng(17).uniform(lo, hi, size=(8, 4096)).astype(np.float32)
    s2 = float(np.float32(s1) / np.float32(255.0))
    xq1, xq2 = oracle.static_quant(x, (s1, z1), (s2, 0))
    d1 = (xq1.astype(np.float64) - z1) * s1
    d2 = xq2.astype(np.float64) * s2
    e1 = np.abs(x - d1).max()
    e2 = np.abs(x - d1 - d2).max()
    assert e1 <= s1 / 2 * (1 + 2.0 ** -18)
    assert e2 <= s1 / 510 * (1 + 2.0 ** -10) + 4 * np.spacing(np.float32(max(abs(lo), hi)))
    assert e2 < e1 / 100


# ------------------------------------------------------------------ linears


def test_int8_to_bf16_cast_is_exact():
    """tiny-llm page: the int8 -> bf16 cast is exact (|q| <= 127 < 256)."""
    q = torch.arange(-128, 128, dtype=torch.int32)
    assert torch.equal(q.to(torch.bfloat16).to(torch.int32), q)


def test_w8a16_factorisation_identity():
    """y = s * (x q^T) equals x dq(W)^T (tiny-llm module docstring) -- numpy fp64 GEMM."""
    x = wl.normal_bf16((5, 96), 1.0, seed=18)
    q, s, _ = oracle.quantize_weight(wl.weight(40, 96, seed=19).numpy())
    y, a = oracle.linear_w8a16(wl.bf16_bits(x), q, s)
    ref = x.double().numpy() @ (q.astype(np.float64) * s.astype(np.float64)[:, None]).T
    assert np.all(np.abs(y - ref) <= 1e-12 * a + 1e-300)
    assert np.abs(y).max() > 0


def test_w8a16_exact_rational_small():
    x = wl.normal_bf16((3, 7), 1.0, seed=20)
    bits = wl.bf16_bits(x)
    q, s, _ = oracle.quantize_weight(wl.weight(5, 7, seed=21).numpy())
    y, _ = oracle.linear_w8a16(bits, q, s)
    for m in range(3):
        for n in range(5):
            exact = sum(bf16_bits_to_fraction(bits[m, k]) * int(q[n, k]) for k in range(7))
            assert y[m, n] == float(exact * f32(s[n]))


def test_w8a16_rows_subset_and_thread_independence():
    x = wl.bf16_bits(wl.normal_bf16((9, 64), 1.0, seed=22))
    q, s, _ = oracle.quantize_weight(wl.weight(33, 64, seed=23).numpy())
    oracle.set_num_threads(1)
    y1, _ = oracle.linear_w8a16(x, q, s)
    oracle.set_num_threads(8)
    y8, _ = oracle.linear_w8a16(x, q, s)
    ys, _ = oracle.linear_w8a16(x, q, s, rows=[7, 2])
    assert np.array_equal(y1, y8)
    assert np.array_equal(ys, y1[[7, 2]])


def test_w8a8_matches_page_forward_and_exact_sums():
    """Q8Linear.forward (SmolVLM q8 page): linear(dq(q(x,s1)), dq(W)) + linear(dq(q(r,s2)), dq(W)),
    evaluated here with numpy fp64 matmuls on the dequantized operands; the raw int32 sums
    against an int64 matmul; and one entry in exact rational arithmetic."""
    x, calib = wl.w8a8_inputs(6, K=64)
    x = x.numpy()
    s1, z1 = oracle.qparams_from_minmax(*oracle.minmax(calib.numpy()))
    s2 = float(np.float32(s1) / np.float32(255.0))
    q, sw, wsum = oracle.quantize_weight(wl.weight(24, 64, seed=24).numpy())
    for second in (None, (s2, 0)):
        y, a, acc1, acc2 = oracle.linear_w8a8(x, (s1, z1), q, sw, second=second)
        xq1, xq2 = oracle.static_quant(x, (s1, z1), second)
        dqw = q.astype(np.float64) * sw.astype(np.float64)[:, None]
        ref = ((xq1.astype(np.float64) - z1) * s1) @ dqw.T
        if second is not None:
            ref += (xq2.astype(np.float64) * s2) @ dqw.T
            assert np.array_equal(acc2, xq2.astype(np.int64) @ q.astype(np.int64).T)
        assert np.all(np.abs(y - ref) <= 1e-12 * a)
        assert np.array_equal(acc1, xq1.astype(np.int64) @ q.astype(np.int64).T)
        t = sum((int(xq1[2, k]) - z1) * int(q[5, k]) for k in range(64))
        ex = f32(s1) * t
        if second is not None:
            ex += f32(s2) * sum(int(xq2[2, k]) * int(q[5, k]) for k in range(64))
        assert abs(Fraction(y[2, 5]) - f32(sw[5]) * ex) <= abs(f32(sw[5]) * ex) * Fraction(1, 2**50)


def test_w8a8_zero_point_term_matters():
    """A nonzero z1 changes y by s_w s1 z1 sum_k q -- the weight_sums correction term."""
    x = wl.normal((2, 32), 1.0, seed=25).numpy()
    q, sw, wsum = oracle.quantize_weight(wl.weight(8, 32, seed=26).numpy())
    s1 = 0.05
    ya, _, acc_a, _ = oracle.linear_w8a8(x, (s1, 0), q, sw)
    yb, _, acc_b, _ = oracle.linear_w8a8(x, (s1, 10), q, sw)
    # codes shift by exactly 10 (no clamping for these magnitudes)
    assert np.array_equal(acc_b - acc_a, 10 * np.broadcast_to(wsum, acc_a.shape))
    assert np.allclose(ya, yb, rtol=1e-12, atol=1e-12)


def test_q4gs_nearest_grid_and_packing():
    W = wl.weight(16, 256, seed=27).numpy()
    for G in (32, 128):
        q4, gs = oracle.quantize_weight_q4gs(W, G)
        lo = (q4 & 0xF).astype(np.int8)
        hi = (q4 >> 4).astype(np.int8)
        codes = np.empty((16, 256), np.int64)
        codes[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
        codes[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
        assert codes.min() >= -7 and codes.max() <= 7
        g = np.repeat(gs.astype(np.float64), G, axis=1)
        assert np.all(np.abs(codes * g - W) <= g * (0.5 + 2.0 ** -20))


def test_dq8ca_q4gsw_reductions():
    """8da4w: (a) against numpy fp64 matmul of (xq - z) and the dequantized weight;
    (b) with G = K and gs = 1 it is s[m] * sum_k (xq - z) q4, an integer matmul."""
    bits = wl.bf16_bits(wl.normal_bf16((5, 128), 1.0, seed=28))
    s, z, xq = oracle.choose_qparams(bits)
    W = wl.weight(12, 128, seed=29).numpy()
    for G in (32, 128):
        q4, gs = oracle.quantize_weight_q4gs(W, G)
        y, a = oracle.linear_dq8ca_q4gsw(xq, s, z, q4, gs, G)
        lo = (q4 & 0xF).astype(np.int64)
        hi = (q4 >> 4).astype(np.int64)
        codes = np.empty((12, 128), np.int64)
        codes[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
        codes[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
        dqw = codes * np.repeat(gs.astype(np.float64), G, axis=1)
        xa = (xq.astype(np.float64) - z[:, None]) * s.astype(np.float64)[:, None]
        ref = xa @ dqw.T
        assert np.all(np.abs(y - ref) <= 1e-12 * a)
        if G == 128:
            ones = np.ones_like(gs)
            y1, _ = oracle.linear_dq8ca_q4gsw(xq, s, z, q4, ones, G)
            ints = (xq.astype(np.int64) - z[:, None]) @ codes.T
            assert np.array_equal(y1, ints * s.astype(np.float64)[:, None])


def test_gemm_s8s8_s32_exact():
    rng = np.random.default_rng(30)
    a = rng.integers(-128, 128, size=(7, 300), dtype=np.int8)
    b = rng.integers(-128, 128, size=(9, 300), dtype=np.int8)
    assert np.array_equal(oracle.gemm_s8s8_s32(a, b), a.astype(np.int64) @ b.astype(np.int64).T)


def test_round_bf16():
    """Once-rounding fp64 -> bf16: torch's fp32 -> bf16 cast on fp32-exact values, ties to even,
    and values that an fp64 -> fp32 -> bf16 double rounding would get wrong."""
    v = wl.normal((1000,), 3.0, seed=31)
    want = wl.bf16_bits(v.to(torch.bfloat16))
    assert np.array_equal(oracle.round_bf16(v.double().numpy()), want)
    one = 1.0
    cases = [one + 2 ** -8, one + 3 * 2 ** -8, -(one + 2 ** -8), one + 2 ** -8 + 2 ** -40]
    got = oracle.round_bf16(np.array(cases))
    exp = [rn_bf16(Fraction(c)) for c in cases]
    assert [bf16_bits_to_fraction(g) for g in got] == exp
    assert got[3] == 0x3F81                          # just above the tie: rounds up


# ------------------------------------------------- full int8 weight grid (f1)


def _weight_codes_full128_exact(row):
    """weight_int8 (SmolVLM q8 page) in exact rational arithmetic with fp32 rounding at
    each step: observer scale max(amax / 127.5, 2^-23), codes clamp(rne(w / s), -128, 127)."""
    vals = [f32(v) for v in row]
    amax = max([Fraction(0)] + [abs(v) for v in vals])
    s = rn32(amax / Fraction(255, 2)) if amax else Fraction(0)
    eps = Fraction(2) ** -23
    if s < eps:
        s = eps
    codes = [max(-128, min(127, rne_int(rn32(v / s)))) for v in vals]
    return s, codes


def test_golden_weight_rows_full128():
    """weight_int8's observer grid (SmolVLM q8 page) on hand-worked rows."""
    rows = _parse("weight_int8_full128_rows.txt")
    W = np.array([[float(v) for v in r[0]] for r in rows], np.float32)
    q, s, ws = oracle.quantize_weight(W, grid="full128")
    for i, r in enumerate(rows):
        assert q[i].tolist() == [int(v) for v in r[2]], f"row {i} codes"
        assert ws[i] == int(r[3][0]), f"row {i} code sum"
        assert s[i] == np.float32(float(r[1][0])), f"row {i} scale"


def test_quantize_weight_full128_exact_rational():
    W = wl.weight(12, 37, seed=31).numpy()
    W[2] = 0.0
    W[4] *= 1e-8                                     # below the eps floor
    W[6, 3] = -np.abs(W[6]).max() * 1.5              # a dominant negative element
    for n in range(W.shape[0]):
        Wn = W[n:n + 1]
        q, s, ws = oracle.quantize_weight(Wn, grid="full128")
        s_ex, codes = _weight_codes_full128_exact(Wn[0])
        assert Fraction(float(s[0])) == s_ex, f"row {n} scale"
        assert q[0].tolist() == codes, f"row {n} codes"
        assert int(ws[0]) == sum(codes)


def test_full128_nearest_grid_and_asymmetric_clamp():
    """|q*s - w| <= s/2 on [-128, 127], up to the rounding of the fp32 quotient w/s (at most
    2^-17 for |w/s| <= 128); the positive extreme never passes 127, and over many rows the
    negative extreme reaches -128 (when amax/127.5 rounds down in fp32) as well as -127
    (when it rounds up)."""
    W = wl.weight(512, 64, seed=32).numpy()
    W[:, 0] = -np.abs(W).max(axis=1) * 1.01          # each row's extreme is negative
    q, s, _ = oracle.quantize_weight(W, grid="full128")
    err = np.abs(q.astype(np.float64) * s[:, None].astype(np.float64) - W.astype(np.float64))
    assert np.all(err <= s[:, None] * (0.5 + 2.0 ** -17))
    assert q.max() <= 127 and q.min() >= -128
    assert (q[:, 0] == -128).any() and (q[:, 0] == -127).any()
    qp, _, _ = oracle.quantize_weight(-W, grid="full128")
    assert np.all(qp[:, 0] == 127)                   # positive extremes clamp at 127


# ------------------------------------------------------------------ bias (f1)


def test_w8a16_bias_closed_form():
    """Int8Linear.forward with a bias (ROCm page: F.linear(x, w, bias)): with q = I and
    s_w = 1 the linear is the identity, so y = x + bias exactly."""
    K = 32
    q = np.eye(K, dtype=np.int8)
    sw = np.ones(K, np.float32)
    xt = wl.normal_bf16((5, K), 1.0, seed=33)
    b = wl.normal((K,), 3.0, seed=34).numpy()
    y, a = oracle.linear_w8a16(wl.bf16_bits(xt), q, sw, bias=b)
    x64 = xt.float().numpy().astype(np.float64)
    assert np.array_equal(y, x64 + b.astype(np.float64)[None, :])
    y0, a0 = oracle.linear_w8a16(wl.bf16_bits(xt), q, sw)
    assert np.array_equal(a - a0, np.broadcast_to(np.abs(b).astype(np.float64), a.shape))


def test_w8a8_bias_first_pass_only():
    """Q8Linear.forward (SmolVLM q8 page) with a bias: linear(dq(q(x)), dq(W), bias) +
    linear(dq(q(r)), dq(W)) -- the bias enters once, also in the two-pass form."""
    x, calib = wl.w8a8_inputs(6, K=64)
    x = x.numpy()
    s1, z1 = oracle.qparams_from_minmax(*oracle.minmax(calib.numpy()))
    s2 = float(np.float32(s1) / np.float32(255.0))
    q, sw, _ = oracle.quantize_weight(wl.weight(24, 64, seed=35).numpy())
    b = wl.normal((24,), 2.0, seed=36).numpy()
    dqw = q.astype(np.float64) * sw.astype(np.float64)[:, None]
    for second in (None, (s2, 0)):
        y, a, _, _ = oracle.linear_w8a8(x, (s1, z1), q, sw, second=second, bias=b)
        xq1, xq2 = oracle.static_quant(x, (s1, z1), second)
        ref = ((xq1.astype(np.float64) - z1) * s1) @ dqw.T + b.astype(np.float64)[None, :]
        if second is not None:
            ref += (xq2.astype(np.float64) * s2) @ dqw.T
        assert np.all(np.abs(y - ref) <= 1e-12 * a)


# ------------------------------------------- residual calibration observer (f2)


def test_golden_residual_observer_rows():
    """calibrate's second run (SmolVLM q8 page) on hand-worked rows."""
    for r in _parse("residual_observer_rows.txt"):
        s1, z1 = float(r[0][0]), int(r[0][1])
        x = np.array([float(v) for v in r[1]], np.float32)
        assert oracle.residual_minmax(x, (s1, z1)) == (float(r[2][0]), float(r[2][1]))


def _residual_exact(x_vals, s1, z1):
    inv = rn32(1 / s1)
    out = []
    for v in x_vals:
        c = max(-128, min(127, rne_int(rn32(v * inv)) + z1))
        out.append(rn32(v - rn32((c - z1) * s1)))
    return out


def test_residual_observer_exact_rational():
    x, calib = wl.w8a8_inputs(3, K=64)
    x = x.numpy().reshape(-1)
    x[5] = 1e4                                       # clamped above
    x[9] = -1e4                                      # clamped below
    for s1, z1 in [(0.05, 3), (float(np.float32(0.0371)), -17), (1.0 / 3.0, 0)]:
        s1 = float(np.float32(s1))
        r = _residual_exact([f32(v) for v in x], f32(s1), z1)
        assert oracle.residual_minmax(x, (s1, z1)) == (float(min(r)), float(max(r)))


def test_residual_observer_half_step_bound():
    """Inside the clamp range the first-pass error is at most half a step (s1/2, up to the
    fp32 rounding of x * (1/s1)); values on the grid leave no residual."""
    s1, z1 = 0.02, 7
    x = wl.normal((4096,), 0.5, seed=37).numpy()      # |x| well inside (-128-7..127-7)*s1
    lo, hi = oracle.residual_minmax(x, (s1, z1))
    assert -s1 * (0.5 + 2.0 ** -16) <= lo <= 0.0 <= hi <= s1 * (0.5 + 2.0 ** -16)
    grid = (np.arange(-100, 100, dtype=np.float32) * np.float32(0.25)).astype(np.float32)
    assert oracle.residual_minmax(grid, (0.25, 0)) == (0.0, 0.0)


# ------------------------------------------------------- GPTQ on the int8 grid (f3)


def _calib_x(R, K, seed, dead=()):
    """Correlated calibration inputs (mixed Gaussian columns), some columns never active."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((R, K))
    mix = np.eye(K) + 0.6 * rng.standard_normal((K, K)) / np.sqrt(K)
    x = (z @ mix).astype(np.float32)
    for k in dead:
        x[:, k] = 0.0
    return x


def test_gram_and_hessian_match_numpy():
    """hessians (SmolVLM q8 page): sum over batches of x^T x in fp64, against numpy's matmul
    (fp32 products are exact in fp64, so only the summation order differs)."""
    x = _calib_x(300, 40, seed=41)
    b1, b2 = x[:170], x[170:]
    H = oracle.hessian([b1, b2])
    ref = b1.astype(np.float64).T @ b1.astype(np.float64) + \
        b2.astype(np.float64).T @ b2.astype(np.float64)
    mag = np.abs(x.astype(np.float64)).T @ np.abs(x.astype(np.float64))
    assert np.all(np.abs(H - ref) <= mag * 300 * 2.0 ** -52)
    assert np.array_equal(oracle.gram(b1, rows=[3, 17]), oracle.gram(b1)[[3, 17]])


def test_gptq_hinv_is_upper_factor_of_damped_inverse():
    K = 48
    x = _calib_x(200, K, seed=42, dead=(5, 30))
    H = oracle.hessian([x])
    U, dead = oracle.gptq_hinv(H, 0.01)
    assert dead.tolist() == [k in (5, 30) for k in range(K)]
    Hd = H.copy()
    Hd[dead, dead] = 1.0
    Hd += 0.01 * np.mean(np.diag(Hd)) * np.eye(K)
    assert np.abs(np.tril(U, -1)).max() == 0.0 and np.all(np.diag(U) > 0)
    assert np.abs(U.T @ U @ Hd - np.eye(K)).max() < 1e-9


def test_gptq_identity_hessian_is_round_to_nearest():
    """With H a multiple of I no error propagates (hinv is diagonal): GPTQ reduces to round
    to nearest on weight_int8's grid and scales -- with the page's float64 division w / s."""
    W = wl.weight(9, 64, seed=43).numpy()
    q, s, ws = oracle.gptq_int8(W, 3.0 * np.eye(64), block=16)
    _, rs, _ = oracle.quantize_weight(W, grid="full128")
    want = np.clip(np.rint(W.astype(np.float64) / rs.astype(np.float64)[:, None]), -128, 127)
    assert np.array_equal(s, rs)
    assert np.array_equal(q, want.astype(np.int8))
    assert np.array_equal(ws, want.sum(axis=1).astype(np.int32))


def _obs_values(w, q, s, Hd):
    """Per column i, the least-squares value of w_i once columns < i are fixed at q * s:
    argmin over u of (w - [q_<i s, u]) Hd (w - [q_<i s, u])^T, solved directly."""
    K = w.size
    v = np.empty(K)
    for i in range(K):
        a = w[:i] - q[:i] * s
        rhs = Hd[i:, :i] @ a
        v[i] = w[i] + np.linalg.solve(Hd[i:, i:], rhs)[0]
    return v


def test_gptq_codes_are_obs_optimal_roundings():
    """Frantar et al.'s result that gptq_int8 implements: the value rounded at column i is
    the optimum of the layer's quadratic error over the not-yet-rounded weights, given the
    codes already chosen.  Checked per column against a direct solve (numpy), away from
    rounding ties."""
    K, N = 20, 4
    x = _calib_x(80, K, seed=44, dead=(3,))
    H = oracle.hessian([x])
    W = wl.weight(N, K, seed=45).numpy() * 50
    _, dead = oracle.gptq_hinv(H)
    Hd = H.copy()
    Hd[dead, dead] = 1.0
    Hd += 0.01 * np.mean(np.diag(Hd)) * np.eye(K)
    for block in (4, 7, 128):                        # ragged last block with 7
        q, s, ws = oracle.gptq_int8(W, H, block=block)
        checked = 0
        for n in range(N):
            w = np.where(dead, 0.0, W[n].astype(np.float64))
            v = _obs_values(w, q[n].astype(np.float64), float(s[n]), Hd) / float(s[n])
            want = np.clip(np.rint(v), -128, 127)
            away = np.abs(np.abs(v - np.floor(v)) - 0.5) > 1e-7
            assert np.array_equal(q[n][away], want[away]), f"row {n} block {block}"
            checked += away.sum()
        assert checked >= 0.95 * N * K
        assert np.array_equal(ws, q.astype(np.int64).sum(axis=1))


def test_gptq_dead_columns_and_error_reduction():
    """Dead columns (never-active inputs) get code 0 even where W is large, and GPTQ's
    quadratic error tr((W - Qs) H (W - Qs)^T) beats round-to-nearest on correlated inputs."""
    K, N = 64, 16
    x = _calib_x(400, K, seed=46, dead=(0, 17))
    H = oracle.hessian([x])
    W = wl.weight(N, K, seed=47).numpy()
    W[:, 17] = 0.05
    q, s, _ = oracle.gptq_int8(W, H, block=16)
    assert not q[:, [0, 17]].any()
    rq, rs, _ = oracle.quantize_weight(W, grid="full128")

    def qerr(codes, sc):
        d = W.astype(np.float64) - codes.astype(np.float64) * sc.astype(np.float64)[:, None]
        return float(np.einsum("nk,kl,nl->", d, H, d))
    assert qerr(q, s) < 0.8 * qerr(rq, rs)


def test_minmax_is_numpy_min_max():
    """act_observer's statistics (SmolVLM q8 page): the min and max of everything observed."""
    x = wl.normal((37, 51), 3.0, seed=48).numpy()
    x[5, 7] = -1e30
    x[36, 50] = 7e29
    assert oracle.minmax(x) == (float(x.min()), float(x.max()))
    assert oracle.minmax(np.full((3,), 2.5, np.float32)) == (2.5, 2.5)


# ------------------------------------------------------ NVFP4 weight-only twin (f4)
# flashrt-structures schemes.py, W4A16Decode: E2M1 codes packed two per byte with a scale
# per 16-element block, bf16 activations.  The format's fields are written out here from
# their bit definitions (not from the oracle) and the oracle is held to them.


def _e2m1_exact(code):
    """E2M1 from its bits: sign 3, exponent 2..1 (bias 1), mantissa 0; exponent 0 is the
    subnormal m * 0.5."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    v = Fraction(m, 2) if e == 0 else Fraction(2) ** (e - 1) * (1 + Fraction(m, 2))
    return -v if s else v


def _e4m3_exact(b):
    """E4M3 from its bits: sign 7, exponent 6..3 (bias 7), mantissa 2..0, subnormals
    m/8 * 2^-6; exponent 15 with mantissa 7 is NaN (None here)."""
    s, e, m = (b >> 7) & 1, (b >> 3) & 15, b & 7
    if e == 15 and m == 7:
        return None
    v = Fraction(m, 8) * Fraction(1, 64) if e == 0 else Fraction(2) ** (e - 7) * (1 + Fraction(m, 8))
    return -v if s else v


def _nearest_code(a, values):
    """Index of the value nearest to a (ties to the even index), saturating at the last."""
    best = 0
    for i, v in enumerate(values):
        d, db = abs(a - v), abs(a - values[best])
        if d < db or (d == db and i % 2 == 0):
            best = i
    if a >= values[-1]:
        best = len(values) - 1
    return best


E2M1_POS = [_e2m1_exact(c) for c in range(8)]
E4M3_POS = [_e4m3_exact(b) for b in range(127)]


def test_e2m1_and_e4m3_tables_exhaustive():
    assert E2M1_POS == [Fraction(v) for v in ("0", "1/2", "1", "3/2", "2", "3", "4", "6")]
    for c in range(16):
        assert Fraction(oracle.e2m1_value(c)) == _e2m1_exact(c), c
    for b in range(256):
        want = _e4m3_exact(b)
        got = oracle.e4m3_value(b)
        if want is None:
            assert np.isnan(got), b
        else:
            assert Fraction(got) == want, b
    assert max(E4M3_POS) == 448 and min(v for v in E4M3_POS if v > 0) == Fraction(1, 512)


def _rn_e2m1_exact(v):
    a = abs(Fraction(float(np.float32(v))))
    c = _nearest_code(a, E2M1_POS)
    return 0 if c == 0 else (8 if v < 0 else 0) | c


def test_rn_e2m1_nearest_even_saturating():
    rng = np.random.default_rng(40)
    vals = list(rng.uniform(-8, 8, 4000).astype(np.float32))
    mids = [(E2M1_POS[i] + E2M1_POS[i + 1]) / 2 for i in range(7)]
    for mid in mids:                                  # exact ties and their neighbours
        f = float(mid)
        vals += [f, -f, np.nextafter(np.float32(f), np.float32(0)),
                 np.nextafter(np.float32(f), np.float32(10))]
    vals += [0.0, -0.0, 6.0, -6.0, 6.5, -100.0, 1e-30, -1e-30]
    for v in vals:
        assert oracle.rn_e2m1(float(v)) == _rn_e2m1_exact(v), v


def test_rn_e4m3_nearest_even_saturating():
    rng = np.random.default_rng(41)
    vals = list(np.exp2(rng.uniform(-12, 10, 3000)).astype(np.float32))
    for i in range(len(E4M3_POS) - 1):
        mid = (E4M3_POS[i] + E4M3_POS[i + 1]) / 2
        f = np.float32(float(mid))
        if Fraction(float(f)) == mid:                 # exact ties (fp32 holds them all)
            vals += [f, np.nextafter(f, np.float32(0)), np.nextafter(f, np.float32(1e4))]
    vals += [0.0, 448.0, 449.0, 464.0, 1e6, 2.0 ** -10, 2.0 ** -9]
    for v in vals:
        a = Fraction(float(np.float32(v)))
        assert oracle.rn_e4m3(float(v)) == _nearest_code(a, E4M3_POS), v


def _nvfp4_golden():
    rows = _parse("nvfp4_blocks.txt")
    blocks = [([float(v) for v in r[0]], int(r[1][0], 16), [int(c, 16) for c in r[2]])
              for r in rows]
    W = np.array([sum((b[0] for b in blocks[0:4]), []), sum((b[0] for b in blocks[4:8]), [])],
                 np.float32)
    return W, blocks


def _unpack_nibbles(q4):
    codes = np.empty((q4.shape[0], 2 * q4.shape[1]), np.int64)
    codes[:, 0::2] = q4 & 0xF
    codes[:, 1::2] = q4 >> 4
    return codes


def test_golden_nvfp4_blocks():
    """Hand-worked blocks: the scale byte and the 16 codes of every block, gsc = 1."""
    W, blocks = _nvfp4_golden()
    q4, sf, gsc = oracle.quantize_weight_nvfp4(W)
    assert gsc == np.float32(1.0)
    codes = _unpack_nibbles(q4)
    for i, (_, e, want) in enumerate(blocks):
        r, b = divmod(i, 4)
        assert sf[r, b] == e, f"block {i} scale"
        assert codes[r, 16 * b:16 * b + 16].tolist() == want, f"block {i} codes"


def test_nvfp4_quantizer_follows_its_steps():
    """Random weights (a zero block, a tiny block, mixed magnitudes): every fp32 step of the
    reading re-done here in exact arithmetic -- the tensor scale, each block's E4M3 byte as
    the nearest to fp32(fp32(amax_b / 6) / gsc), each code as the nearest E2M1 to
    fp32(w / d) with d = fp32(e4m3 * gsc)."""
    W = wl.weight(6, 256, seed=42).numpy()
    W[1, 16:32] = 0.0
    W[2, 32:48] *= 1e-6
    W[3] *= 50.0
    q4, sf, gsc = oracle.quantize_weight_nvfp4(W)
    assert gsc == np.float32(np.abs(W).max()) / np.float32(2688.0)
    codes = _unpack_nibbles(q4)
    for n in range(W.shape[0]):
        for b in range(16):
            blk = W[n, 16 * b:16 * b + 16]
            sb = np.float32(np.abs(blk).max()) / np.float32(6.0)
            e = _nearest_code(Fraction(float(np.float32(sb / gsc))), E4M3_POS)
            assert sf[n, b] == e, (n, b)
            d = np.float32(np.float32(float(_e4m3_exact(e))) * gsc)
            for j in range(16):
                want = 0 if d == 0 else _rn_e2m1_exact(np.float32(blk[j] / d))
                assert codes[n, 16 * b + j] == want, (n, b, j)


def test_w4a16_nvfp4_factorisation_identity():
    """The linear is gsc * x . (e2m1 * e4m3): a numpy fp64 matmul on weights decoded here."""
    bits = wl.bf16_bits(wl.normal_bf16((5, 256), 1.0, seed=43))
    W = wl.weight(9, 256, seed=44).numpy()
    W[4, :16] = 0.0
    q4, sf, gsc = oracle.quantize_weight_nvfp4(W)
    codes = _unpack_nibbles(q4)
    dq = np.array([[float(_e2m1_exact(int(codes[n, k])) * _e4m3_exact(int(sf[n, k // 16])))
                    for k in range(256)] for n in range(9)])
    x = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = (x @ dq.T) * float(gsc)
    y, a = oracle.linear_w4a16_nvfp4(bits, q4, sf, gsc)
    assert np.all(np.abs(y - ref) <= 1e-12 * a + 1e-300)
    y2, _ = oracle.linear_w4a16_nvfp4(bits, q4, sf, gsc, rows=[4, 0])
    assert np.array_equal(y2, y[[4, 0]])
    # dequantized weights stay within half a grid step (plus saturation) of W
    assert np.all(np.abs(dq * float(gsc) - W) <= np.abs(W).max() / 6 * 1.0 + 1e-30)
