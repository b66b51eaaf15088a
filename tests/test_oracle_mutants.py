"""Mutation gate for the oracle's pins (CPU only).

Each mutant is a copy of the oracle's C source with one plausible mistake
planted in it (the kind of defect that gives fluent wrong numbers instead of a
crash).  The copy is compiled into a temporary directory and the pins are run
against it: at least one pin must fail, or the pins would not have caught that
mistake in the real oracle either.
"""
import os

import pytest

import oracle as oracle_pkg
import oracle_pins as P

# (name, text in the oracle source, replacement)
MUTANTS = [
    ("nibble_order_reversed", "(word >> (4 * (k % 8)))", "(word >> (4 * (7 - k % 8)))"),
    ("scale_group_off_by_one", "scales[n * (K / group) + k / group]",
     "scales[n * (K / group) + (k / group + 1) % (K / group)]"),
    ("scale_group_fixed_32", "scales[n * (K / group) + k / group]",
     "scales[n * (K / group) + (k / ZTO_GROUP) % (K / group)]"),
    ("zero_point_8", "#define ZTO_ZERO 7", "#define ZTO_ZERO 8"),
    ("gate_up_swapped",
     "double g = zto_row_dot(qw, scales, x, K, group, m, n);",
     "double g = zto_row_dot(qw, scales, x, K, group, m, n + N);"),
    ("argmax_highest_index_on_tie", "if (c > best_v) {", "if (c >= best_v) {"),
    ("dropped_k_tail", "for (int64_t k = 0; k < K; ++k)\n        acc +=",
     "for (int64_t k = 0; k < K - 1; ++k)\n        acc +="),
    ("half_exponent_bias", "expo - 25", "expo - 24"),
    ("half_subnormal_scale", "ldexp((double)frac, -24)", "ldexp((double)frac, -25)"),
    ("silu_sign", "return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));"),
    ("argmax_leading_nan_wins", "double best_v = isnan(v[0]) ? -INFINITY : v[0];",
     "double best_v = v[0];"),
    ("pack_high_nibble_first", "word |= (uint32_t)c << (4 * j);",
     "word |= (uint32_t)c << (4 * (7 - j));"),
    ("x_row_stride", "zto_weight(qw, scales, K, group, n, k) * zto_half_to_double(x[m * K + k])",
     "zto_weight(qw, scales, K, group, n, k) * zto_half_to_double(x[k])"),
    ("rmsnorm_eps_outside_sqrt", "1.0 / sqrt(ss / (double)K + eps)", "1.0 / (sqrt(ss / (double)K) + eps)"),
    ("rmsnorm_sum_not_mean", "1.0 / sqrt(ss / (double)K + eps)", "1.0 / sqrt(ss + eps)"),
    ("rmsnorm_gamma_dropped", "hd * r * zto_half_to_double(gamma[k])", "hd * r"),
    ("rmsnorm_gamma_reversed", "hd * r * zto_half_to_double(gamma[k])", "hd * r * zto_half_to_double(gamma[K - 1 - k])"),
    ("rmsnorm_delta_ignored_in_h", "if (h_out) h_out[m * K + k] = hb;",
     "if (h_out) h_out[m * K + k] = residual[m * K + k];"),
    ("rmsnorm_rows_share_one_sum", "    for (int64_t m = 0; m < M; ++m) {\n        double ss = 0.0;",
     "    double ss = 0.0;\n    for (int64_t m = 0; m < M; ++m) {"),
    ("half_rounding_ties_away", "(frac == 0.5 && fmod(r, 2.0) != 0.0)", "(frac == 0.5)"),
    ("half_subnormal_spacing", "if (e < -14) e = -14;", "if (e < -15) e = -15;"),
    ("rope_neighbour_pairs", "const int64_t n = h * head_dim + i, n2 = n + half;",
     "const int64_t n = h * head_dim + 2 * i, n2 = n + 1;"),
    ("rope_sin_sign", "out[m * N + n] = a * cos(phi) - b * sin(phi);", "out[m * N + n] = a * cos(phi) + b * sin(phi);"),
    ("rope_frequency_exponent", "pow(theta, -2.0 * (double)i / (double)head_dim)", "pow(theta, -(double)i / (double)head_dim)"),
    ("rope_first_token_position", "const double phi = (double)pos[m] * inv_freq;", "const double phi = (double)pos[0] * inv_freq;"),
    ("gemm_f16w_weights_not_rounded",
     "w[k] = zto_half_to_double(zto_double_to_half(zto_weight(qw, scales, K, group, n, k)));",
     "w[k] = zto_weight(qw, scales, K, group, n, k);"),
    ("dequant_f16_transposed", "w16[n * K + k] = zto_double_to_half", "w16[k * N + n] = zto_double_to_half"),
    ("gemm_f16w_first_token_for_all", "acc += w[k] * zto_half_to_double(x[m * K + k]);",
     "acc += w[k] * zto_half_to_double(x[k]);"),
    ("gemm_f16w_rows_ignored", "const int64_t n = rows ? rows[i] : i;\n        double *w = ",
     "const int64_t n = i;\n        double *w = "),
    ("gate_up_f16w_rows_ignored", "const int64_t n = rows ? rows[i] : i;\n        double *wg = ",
     "const int64_t n = i;\n        double *wg = "),
    ("gate_up_f16w_up_is_gate", "zto_weight(qw, scales, K, group, N + n, k)", "zto_weight(qw, scales, K, group, n, k)"),
    ("gate_up_f16w_weights_not_rounded",
     "wg[k] = zto_half_to_double(zto_double_to_half(zto_weight(qw, scales, K, group, n, k)));",
     "wg[k] = zto_weight(qw, scales, K, group, n, k);"),
    ("sampled_rows_ignored", "int64_t n = rows ? rows[i] : i;\n        for (int64_t m = 0; m < M; ++m)\n            y[",
     "int64_t n = i;\n        for (int64_t m = 0; m < M; ++m)\n            y["),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    with open(oracle_pkg.SOURCE) as fh:
        src = fh.read()
    assert src.count(old) == 1, f"mutation site for {name} must occur exactly once"
    mutated = tmp_path / f"mutant_{name}.c"
    mutated.write_text(src.replace(old, new))
    lib = oracle_pkg.compile_oracle(str(mutated), str(tmp_path / f"lib_{name}.so"))
    mutant = oracle_pkg.Oracle(lib)
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
