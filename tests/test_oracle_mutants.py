"""Each planted mistake in a copy of the oracle must fail at least one pin.

The mistakes are the plausible ones: a dropped term, a wrong sign, index or
operand order, a wrong rounding mode, a wrong constant.  Every mutant is a
textual edit of ``oracle/bitnet_oracle.c`` compiled into a temporary library;
all edits keep every memory access in bounds.
"""
import os

import pytest

import oracle
import oracle_pins
from oracle import build as oracle_build

MUTANTS = {
    "round_half_away": ("float q = nearbyintf(prod);", "float q = roundf(prod);"),
    "scale_128": ("const float scale = 127.0f / denom;", "const float scale = 128.0f / denom;"),
    "scale_inverted": ("float prod = row[k] * scale;", "float prod = row[k] / scale;"),
    "amax_floor_1e-3": ("amax > ORACLE_QUANT_EPS ? amax : ORACLE_QUANT_EPS",
                        "amax > 1e-3f ? amax : 1e-3f"),
    "amax_not_abs": ("float a = fabsf(row[k]);", "float a = row[k];"),
    "rowsum_abs": ("sum += (int64_t)q;", "sum += (int64_t)fabsf(q);"),
    # (a clamp at -127 instead of -128 would be an equivalent mutant: |x*s| <= 127)
    "clamp_high_126": ("if (q > 127.0f) q = 127.0f;", "if (q > 126.0f) q = 126.0f;"),
    "gamma_no_abs": ("row += fabs((double)w[n * k_cols + k]);", "row += (double)w[n * k_cols + k];"),
    "gamma_rows_only": ("return total / (double)(n_rows * k_cols);", "return total / (double)(k_cols);"),
    "eps_dropped": ("const float d = gamma + eps;", "const float d = gamma;"),
    "ternary_no_clamp": ("if (q > 1.0f) q = 1.0f;", ""),
    "ternary_trunc": ("float q = nearbyintf(w[i] / d);", "float q = truncf(w[i] / d);"),
    "pack_b_j_swapped": ("packed[n * row_bytes + 4 * group + b] |= (uint8_t)(code << (2 * j));",
                         "packed[n * row_bytes + 4 * group + j] |= (uint8_t)(code << (2 * b));"),
    "pack_offset_2": ("uint8_t code = (uint8_t)(w_q[n * k_cols + k] + 1);",
                      "uint8_t code = (uint8_t)(w_q[n * k_cols + k] + 2);"),
    "unpack_wrong_shift": ("int code = (packed[n * row_bytes + 4 * group + b] >> (2 * j)) & 3;",
                           "int code = (packed[n * row_bytes + 4 * group + b] >> (2 * b)) & 3;"),
    "matmul_k_reversed": ("sum += (int64_t)x_q[m * k_cols + k] * (int64_t)w_q[n * k_cols + k];",
                          "sum += (int64_t)x_q[m * k_cols + (k_cols - 1 - k)] * (int64_t)w_q[n * k_cols + k];"),
    "matmul_int8_wrap": ("sum += (int64_t)x_q[m * k_cols + k] * (int64_t)w_q[n * k_cols + k];",
                         "sum = (int8_t)(sum + x_q[m * k_cols + k] * w_q[n * k_cols + k]);"),
    "dequant_scale_inverted": ("(double)gamma / (double)s[m];", "(double)s[m] / (double)gamma;"),
    "dequant_first_row_scale": ("(double)gamma / (double)s[m];", "(double)gamma / (double)s[0];"),
    "relu_dropped": ("double r = g[i] > 0.0 ? g[i] : 0.0;", "double r = g[i];"),
    "relu_not_squared": ("h[i] = r * r * u[i];", "h[i] = r * u[i];"),
    "bf16_shift": ("uint32_t bits = ((uint32_t)src[i]) << 16;", "uint32_t bits = ((uint32_t)src[i]) << 15;"),
    "rms_eps_dropped": ("1.0 / sqrt(ss / (double)k_cols + (double)eps)", "1.0 / sqrt(ss / (double)k_cols)"),
    "rms_mean_k_minus_1": ("1.0 / sqrt(ss / (double)k_cols + (double)eps)",
                           "1.0 / sqrt(ss / (double)(k_cols - 1) + (double)eps)"),
    "rms_not_inverted": ("(float)(1.0 / sqrt(ss / (double)k_cols + (double)eps));",
                         "(float)(sqrt(ss / (double)k_cols + (double)eps));"),
    "rms_weight_dropped": ("y[m * k_cols + k] = xr * g[k];", "y[m * k_cols + k] = xr;"),
    "rms_weight_first_only": ("y[m * k_cols + k] = xr * g[k];", "y[m * k_cols + k] = xr * g[0];"),
    # sum of squares: any fixed binary64 order, a wrong rounding, a lost carry or exponent
    "sumsq_forward_binary64": ("return ss_round(acc);",
                               "double f = 0.0; for (int64_t k = 0; k < k_cols; ++k) f += (double)row[k] * (double)row[k]; return f;"),
    "sumsq_reverse_binary64": ("return ss_round(acc);",
                               "double f = 0.0; for (int64_t k = k_cols - 1; k >= 0; --k) f += (double)row[k] * (double)row[k]; return f;"),
    "sumsq_strided_partials": ("return ss_round(acc);",
                               "double pt[256] = {0}; for (int64_t k = 0; k < k_cols; ++k) pt[k % 256] += (double)row[k] * (double)row[k]; "
                               "double f = 0.0; for (int t = 0; t < 256; ++t) f += pt[t]; return f;"),
    "sumsq_ties_away": ("if (round && (sticky || (mant & 1u))) mant += 1;", "if (round) mant += 1;"),
    "sumsq_truncates": ("if (round && (sticky || (mant & 1u))) mant += 1;", ""),
    "sumsq_sticky_dropped": ("if (round && (sticky || (mant & 1u)))", "if (round && (mant & 1u))"),
    "sumsq_carry_lost": ("carry = t >> 32;", "carry = 0;"),
    "sumsq_subnormal_hidden_bit": ("(field ? 0x800000u : 0u)", "0x800000u"),
    "sumsq_exponent_off": ("ss_add(acc, mant * mant, 2 * e - 2);", "ss_add(acc, mant * mant, 2 * e);"),
    "sumsq_abs_not_square": ("ss_add(acc, mant * mant, 2 * e - 2);", "ss_add(acc, mant, e + 149);"),
    "bf16_truncate": ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;", ""),
    "bf16_ties_away": ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;",
                       "if (lower >= 0x8000u) upper += 1u;"),
    "bf16_ties_odd": ("(lower == 0x8000u && (upper & 1u))", "(lower == 0x8000u && !(upper & 1u))"),
    "bf16_nan_unquieted": ("if ((bits & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((bits >> 16) | 0x0040u);", ""),
    "epi_scale_inverted": ("const float rg = gamma_g / s[m];", "const float rg = s[m] / gamma_g;"),
    "epi_binary64_product": ("const float g = (float)acc_g[i] * rg;",
                             "const float g = (float)((double)acc_g[i] * (double)gamma_g / (double)s[m]);"),
    "epi_relu_dropped": ("const float p = g > 0.0f ? g : 0.0f;", "const float p = g;"),
    "epi_up_uses_gate_gamma": ("const float ru = gamma_u / s[m];", "const float ru = gamma_g / s[m];"),
    "epi_not_squared": ("const float pp = p * p;", "const float pp = p;"),
    "absmax_signed": ("const float a = fabsf(v[m * n_rows + n]);", "const float a = v[m * n_rows + n];"),
    "absmax_first_column": ("const float a = fabsf(v[m * n_rows + n]);", "const float a = fabsf(v[m * n_rows]);"),
    "given_amax_ignored": ("if (amax_in) amax = amax_in[m];", ""),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle_build.SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    path = tmp_path / "mutant.c"
    path.write_text(mutated)
    lib = oracle._bind(oracle_build.compile_source(str(path), str(tmp_path / f"lib_{name}.so")))
    saved = oracle._load()
    oracle._lib = lib
    failed = []
    try:
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except AssertionError:
                failed.append(pin.__name__)
    finally:
        oracle._lib = saved
    assert failed, f"mutant {name} passed every pin"
