"""Mutation checks for the oracle's pins: each case plants one plausible mistake in a copy
of the oracle source (on the CPU), rebuilds it, and requires that at least one pin fails.
This shows the pins would catch that mistake in the real oracle."""
import os
import subprocess

import pytest

import oracle
import oracle.build as ob
import test_oracle_pins as pins

MUTANTS = [
    # (name, text in q8_oracle.c, replacement, pins that must catch it)
    ("ties away from zero (weights)", "float r = nearbyintf(w[k] / scale);   /* true",
     "float r = roundf(w[k] / scale);   /* true", ["test_golden_weight_rows"]),
    ("reciprocal instead of division (weights)", "float r = nearbyintf(w[k] / scale);   /* true",
     "float r = nearbyintf(w[k] * (1.0f / scale));   /* true",
     ["test_weight_codes_divide_not_reciprocal"]),
    ("zero row keeps scale 0", "if (zero) scale = 1.0f;\n        int64_t sum",
     "if (zero) scale = 0.0f;\n        int64_t sum", ["test_zero_row_rule_and_clamp"]),
    ("row max instead of absmax", "float a = fabsf(w[k]);\n            if (a > amax) amax = a;\n        }\n        float scale = amax / 127.0f;",
     "float a = w[k];\n            if (a > amax) amax = a;\n        }\n        float scale = amax / 127.0f;",
     ["test_golden_weight_rows"]),
    ("range not widened to 0", "if (mn > 0.0f) mn = 0.0f;", "",
     ["test_qparams_from_minmax_matches_row_rule"]),
    ("zero point sign", "float zf = -128.0f - nearbyintf(mn / scale);",
     "float zf = -128.0f + nearbyintf(mn / scale);", ["test_golden_activation_rows"]),
    ("divide activations by s", "float t = x * inv;", "float t = x / (1.0f / inv);",
     ["test_activation_codes_multiply_by_reciprocal"]),
    ("residual sign", "float r = x[i] - d1;", "float r = d1 - x[i];",
     ["test_static_codes_use_fp32_reciprocal"]),
    ("w8a8 drops the zero point", "t1 += ((int64_t)c1[k] - z1) * w;", "t1 += (int64_t)c1[k] * w;",
     ["test_w8a8_matches_page_forward_and_exact_sums"]),
    ("w8a8 second pass dropped", "v += (double)s2 * (double)t2;", "v += 0.0;",
     ["test_w8a8_matches_page_forward_and_exact_sums"]),
    ("w8a16 scale of wrong row", "y[i * N + n] = acc * (double)s_w[n];",
     "y[i * N + n] = acc * (double)s_w[(n + 1) % N];", ["test_w8a16_factorisation_identity"]),
    ("w8a16 transposed weight index", "(double)bf16_to_f32(xr[k]) * (double)qr[k];",
     "(double)bf16_to_f32(xr[k]) * (double)q[k * N + n];",
     ["test_w8a16_factorisation_identity"]),
    ("q4 nibble order swapped", "if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | nib);",
     "if ((k & 1) == 1) *byte = (uint8_t)((*byte & 0xF0) | nib);",
     ["test_golden_q4_groups"]),
    ("q4 group scale index", "acc += (double)gs[n * ng + g] * (double)part;",
     "acc += (double)gs[n * ng] * (double)part;", ["test_dq8ca_q4gsw_reductions"]),
    ("q4 zero point dropped", "int64_t p = ((int64_t)xr[k] - z[m]) * q4_code(wr, k);",
     "int64_t p = ((int64_t)xr[k]) * q4_code(wr, k);", ["test_dq8ca_q4gsw_reductions"]),
    ("zero fold drops the group scale", "acc += (double)part * (double)gs[n * ng + g];",
     "acc += (double)part;", ["test_golden_q4gs_zero_fold"]),
    ("zero fold skips the last group", "for (int64_t g = 0; g < ng; ++g) {\n            int64_t part = 0;\n            for (int64_t k = g * G; k < (g + 1) * G; ++k) part +=",
     "for (int64_t g = 0; g < ng - 1; ++g) {\n            int64_t part = 0;\n            for (int64_t k = g * G; k < (g + 1) * G; ++k) part +=",
     ["test_q4gs_zero_fold_exact_row_sums"]),
    ("e2m1 ties away from zero", "if (dc < db || (dc == db && (c & 1) == 0)) best = c;",
     "if (dc <= db) best = c;", ["test_rn_e2m1_nearest_even_saturating"]),
    ("e4m3 rounding truncates", "if (d < bd || (d == bd && (b & 1) == 0)) {",
     "if ((double)q8o_e4m3_value(b) <= (double)v) {", ["test_rn_e4m3_nearest_even_saturating"]),
    ("nvfp4 block scale amax/4", "const float sb = bmax / 6.0f;", "const float sb = bmax / 4.0f;",
     ["test_golden_nvfp4_blocks"]),
    ("nvfp4 tensor scale over 448", "float gsc = amax / 2688.0f;", "float gsc = amax / 448.0f;",
     ["test_golden_nvfp4_blocks"]),
    ("nvfp4 nibble order", "if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | code);",
     "if ((k & 1) == 1) *byte = (uint8_t)((*byte & 0xF0) | code);", ["test_golden_nvfp4_blocks"]),
    ("w4a16 scale of the next block", "(double)q8o_e4m3_value(sf[n * nb + k / 16]);",
     "(double)q8o_e4m3_value(sf[n * nb + (k / 16 + 1) % nb]);",
     ["test_w4a16_nvfp4_factorisation_identity"]),
    ("bf16 rounding truncates", "double r = nearbyint(ldexp(m, 8));",
     "double r = trunc(ldexp(m, 8));", ["test_round_bf16"]),
    ("full grid clamps at -127",
     "r = clampf(r, -128.0f, 127.0f);\n            const int code = (int)r;",
     "r = clampf(r, -127.0f, 127.0f);\n            const int code = (int)r;",
     ["test_golden_weight_rows_full128"]),
    ("full grid scale amax/127", "float scale = amax / half_range;",
     "float scale = amax / 127.0f;", ["test_golden_weight_rows_full128"]),
    ("full grid eps floor only for a zero scale",
     "float scale = amax / half_range;\n        if (scale < FLT_EPSILON) scale = FLT_EPSILON;",
     "float scale = amax / half_range;\n        if (scale == 0.0f) scale = FLT_EPSILON;",
     ["test_golden_weight_rows_full128"]),
    ("residual observer without the clamp",
     "float q = clampf(nearbyintf(x[i] * inv) + (float)z1, -128.0f, 127.0f);",
     "float q = nearbyintf(x[i] * inv) + (float)z1;", ["test_golden_residual_observer_rows"]),
    ("residual observer sign", "float r = x[i] - fq;", "float r = fq - x[i];",
     ["test_golden_residual_observer_rows"]),
    ("residual observer drops the zero point", "float fq = (q - (float)z1) * s1;",
     "float fq = q * s1;", ["test_golden_residual_observer_rows"]),
    ("gptq error not scaled by the inverse-Hessian pivot",
     "const double e = (col - qc * sd) / U[i * K + i];", "const double e = (col - qc * sd);",
     ["test_gptq_codes_are_obs_optimal_roundings"]),
    ("gptq block update sign", "w[j] = w[j] - p;", "w[j] = w[j] + p;",
     ["test_gptq_codes_are_obs_optimal_roundings"]),
    ("gptq damping on every entry",
     "for (int64_t k = 0; k < K; ++k) H[k * K + k] = H[k * K + k] + add;",
     "for (int64_t k = 0; k < K * K; ++k) H[k] = H[k] + add;",
     ["test_gptq_hinv_is_upper_factor_of_damped_inverse"]),
    ("gptq dead column kept", "w[k] = dead[k] ? 0.0 : (double)wrow[k];",
     "w[k] = (double)wrow[k];", ["test_gptq_dead_columns_and_error_reduction"]),
    ("gptq lower factor instead of upper", "U[i * K + j] = L[j * K + i];",
     "U[i * K + j] = L[i * K + j];", ["test_gptq_hinv_is_upper_factor_of_damped_inverse"]),
    ("gram drops the last calibration row", "for (int64_t t = 0; t < R; ++t) {\n            const double xi",
     "for (int64_t t = 0; t < R - 1; ++t) {\n            const double xi",
     ["test_gram_and_hessian_match_numpy"]),
    ("full grid ignores negative extremes", "const float amax = (-lo > hi) ? -lo : hi;",
     "const float amax = hi;", ["test_golden_weight_rows_full128"]),
]


@pytest.mark.parametrize("name,old,new,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new, catchers):
    src = open(ob.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique/found: {old!r}"
    mut = tmp_path / "q8_oracle.c"
    mut.write_text(src.replace(old, new))
    (tmp_path / "q8_oracle.h").write_text(open(os.path.join(ob.HERE, "q8_oracle.h")).read())
    so = str(tmp_path / "libmut.so")
    subprocess.check_call(["gcc", *ob.CFLAGS, str(mut), "-o", so, "-lm"])
    caught = []
    with oracle.use_library(so):
        for fn in catchers:
            try:
                getattr(pins, fn)()
            except AssertionError:
                caught.append(fn)
    assert caught, f"mutant '{name}' survived pins {catchers}"
