"""The oracle's pins must catch plausible mistakes.

Each case below plants one mistake in a copy of the oracle's C source (on the
CPU, never in the committed file), builds it, and checks that at least one pin
of tests/test_oracle.py fails against it.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
import oracle.oracle as oracle_mod
from tests import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle_mod.__file__), "sherry_oracle.c")

MUTANTS = {
    "tie_to_highest_index": ("if (fabsf(w[i]) < fabsf(w[p])) p = i;",
                             "if (fabsf(w[i]) <= fabsf(w[p])) p = i;"),
    "nonpositive_is_negative": ("neg[r++] = (w[i] < 0.0f) ? 1 : 0;",
                                "neg[r++] = (w[i] <= 0.0f) ? 1 : 0;"),
    "zero_words_split_by_half": ("z[j & 1] |= (uint32_t)p << (2 * (j >> 1));",
                                 "z[j >> 4] |= (uint32_t)p << (2 * (j & 15));"),
    "unpack_sign_bit_off_by_one": ("v = ((s[r] >> j) & 1u) ? -1 : 1;",
                                   "v = ((s[r] >> ((j + 1) & 31)) & 1u) ? -1 : 1;"),
    "unpack_ranks_reversed": ("v = ((s[r] >> j) & 1u) ? -1 : 1;",
                              "v = ((s[2 - r] >> j) & 1u) ? -1 : 1;"),
    "scale_over_all_weights": ("scales[n] = (float)(sum_abs / (0.75 * (double)K));",
                               "scales[n] = (float)(sum_abs / (double)K);"),
    "scale_includes_zeroed": ("if (i != p) sum_abs += fabs((double)blk[i]);",
                              "sum_abs += fabs((double)blk[i]) * 0.75;"),
    "dot_drops_last_term": ("for (int64_t k = 0; k < K; k++) a += (int64_t)row[k] * (int64_t)xm[k];",
                            "for (int64_t k = 0; k + 1 < K; k++) a += (int64_t)row[k] * (int64_t)xm[k];"),
    "dot_transposed_activation": ("const int8_t *xm = x + m * K;",
                                  "const int8_t *xm = x + (M - 1 - m) * K;"),
    "y_without_scale": ("y[m * N + n] = (double)scales[n] * (double)acc[m * N + n];",
                        "y[m * N + n] = (double)acc[m * N + n];"),
    "planes_swapped": ("codes[orc_word(2, n, t, T)] = s[0];\n            codes[orc_word(3, n, t, T)] = s[1];",
                       "codes[orc_word(3, n, t, T)] = s[0];\n            codes[orc_word(2, n, t, T)] = s[1];"),
    "group_of_16_rows": ("return ((n / ORC_GROUP) * T + t) * (ORC_NPLANE * ORC_GROUP) + plane * ORC_GROUP + n % ORC_GROUP;",
                         "return ((n / 16) * T + t) * (ORC_NPLANE * 16) + plane * 16 + n % 16;"),
    "rows_before_tiles": ("return ((n / ORC_GROUP) * T + t) * (ORC_NPLANE * ORC_GROUP) + plane * ORC_GROUP + n % ORC_GROUP;",
                          "return ((n / ORC_GROUP) * T + t) * (ORC_NPLANE * ORC_GROUP) + (n % ORC_GROUP) * ORC_NPLANE + plane;"),
    "quantize_truncates": ("float r = nearbyintf(v);", "float r = truncf(v);"),
    "quantize_ties_away": ("float r = nearbyintf(v);", "float r = roundf(v);"),
    "quantize_scale_over_128": ("*s = amax / 127.0f;", "*s = amax / 128.0f;"),
    "quantize_inverse_scale_128": ("const float inv = 127.0f / amax;", "const float inv = 128.0f / amax;"),
    "quantize_f32_reads_row_0": ("orc_quantize_row(x + b * K, K, q + b * K, s + b);",
                                 "orc_quantize_row(x, K, q + b * K, s + b);"),
    "swiglu_exp_of_plus_g": ("gd / (1.0 + exp(-gd))", "gd / (1.0 + exp(gd))"),
    "swiglu_drops_up": ("gd / (1.0 + exp(-gd)) * (double)u[i]", "gd / (1.0 + exp(-gd))"),
    "swiglu_sigmoid_only": ("gd / (1.0 + exp(-gd)) * (double)u[i]", "1.0 / (1.0 + exp(-gd)) * (double)u[i]"),
    "act_scale_dropped": ("y[b * N + n] = (double)scales[n] * (double)sx[b] * (double)acc[b * N + n];",
                          "y[b * N + n] = (double)scales[n] * (double)acc[b * N + n];"),
}


def _run_pins(golden_dir):
    """Return True when every pin passes."""
    checks = [
        pins.test_code_space_is_exactly_32_blocks,
        lambda: pins.test_prune_cases(golden_dir),
        lambda: pins.test_golden_tiles(golden_dir),
        lambda: pins.test_golden_words_unpack_without_pack(golden_dir),
        lambda: pins.test_blocked_layout_across_rows_and_tiles(golden_dir),
        pins.test_pack_unpack_roundtrip_and_scale,
        pins.test_all_ones_activation_gives_sum_of_signs,
        lambda: pins.test_bruteforce_dense_matmul(3, 256, 2),
        lambda: pins.test_bruteforce_dense_matmul(17, 640, 5),
        pins.test_quantize_act_hand_cases,
        pins.test_quantize_act_bounds_on_random_rows,
        pins.test_gemv_act_equals_scaled_bruteforce,
        pins.test_quantize_f32_hand_cases,
        pins.test_quantize_f32_bounds_on_random_rows,
        pins.test_swiglu_closed_forms,
        pins.test_swiglu_minimum_is_lambert_w,
    ]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, golden_dir):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "m.c")
        so = os.path.join(d, "libm_%s.so" % name)
        with open(c, "w") as f:
            f.write(src.replace(old, new))
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", so, c])
        try:
            oracle_mod.use_library(so)
            assert not _run_pins(golden_dir), "pins did not catch mutant " + name
        finally:
            oracle_mod.use_library(None)


def test_committed_oracle_passes(golden_dir):
    assert _run_pins(golden_dir)
