"""Plant mistakes in copies of the oracle's C file and check that the pins
catch every one: evidence that the pins constrain each step of the oracle
(rounding, scale, zero point, range widening, clamp, packing map, decoding,
linear indexing).  Everything runs on the CPU."""
from __future__ import annotations

import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as O
import tests.test_oracle_pins as P

MUTANTS = {
    "round_half_away": ("int r = (int)nearbyintf(t);", "int r = (int)roundf(t);"),
    "zero_round_half_away": ("int z = (int)nearbyintf(zq);", "int z = (int)roundf(zq);"),
    "levels_2^b": ("float s = range / (float)qmax;", "float s = range / (float)(qmax + 1);"),
    "no_zero_in_range": ("if (lo > 0.0f) lo = 0.0f;", ""),
    "zero_sign": ("float zq = -lo / s;", "float zq = lo / s;"),
    "reciprocal_multiply": ("float t = x[i] / s;", "float t = x[i] * (1.0f / s);"),
    "no_clamp": ("if (q > qmax) q = qmax;", ""),
    "lane_transposed": ("int lane = 4 * r + c;", "int lane = 4 * c + r;"),
    "nibble_pairing": ("field = slot + 4 * odd;", "field = 2 * slot + odd;"),
    "crumb_run_offset": ("field = 4 * (run % 2) + slot + 8 * odd;", "field = 8 * (run % 2) + slot + 4 * odd;"),
    "linear_zero_sign": ("wrow[k] = (double)((int)codes[n * K + k] - (int)zeros[n * G + j])",
                         "wrow[k] = (double)((int)codes[n * K + k] + (int)zeros[n * G + j])"),
    "linear_scale_transposed": ("* (double)scales[n * G + j];\n        }\n        for (int64_t m",
                                "* (double)scales[j * N + n];\n        }\n        for (int64_t m"),
    "meta_row_major": ("return 128 * G * (n / 128) + g * block_rows(n, rows) + n % 128;",
                       "return 128 * G * (n / 128) + g * 128 + n % 128;"),
    "tile_order_row_major": ("*byte_off = block_start + (kt * Rb + t) * 512", "*byte_off = block_start + (t * (cols / T) + kt) * 512"),
    "f16_bias": ("mag = ldexpf((float)(1024 + f), e - 25);", "mag = ldexpf((float)(1024 + f), e - 24);"),
    "f16_subnormal": ("mag = ldexpf((float)f, -24);", "mag = ldexpf((float)f, -25);"),
    "sym_levels_2^b-1": ("float s = amax / (float)(z - 1);", "float s = amax / (float)qmax;"),
    "sym_no_offset": ("int q = (int)nearbyintf(x[i] / s) + z;", "int q = (int)nearbyintf(x[i] / s);"),
    "sym_round_half_away": ("int q = (int)nearbyintf(x[i] / s) + z;", "int q = (int)roundf(x[i] / s) + z;"),
    "sym_min_not_abs": ("float a = fabsf(x[i]);", "float a = x[i];"),
    "grad_zero_sign": ("wcol[n] = (double)((int)codes[n * K + k] - (int)zeros[n * G + j])",
                       "wcol[n] = (double)((int)codes[n * K + k] + (int)zeros[n * G + j])"),
    "grad_dy_transposed": ("acc += dy[m * N + n] * wcol[n];", "acc += dy[n * M + m] * wcol[n];"),
    "grad_group_of_column": ("const int64_t j = k / group;", "const int64_t j = (k / group) % (G > 1 ? G - 1 : 1);"),
    "dequant32_zero_sign": ("float d = (float)((int)codes[n * cols + k] - (int)zeros[n * G + j]);",
                            "float d = (float)((int)codes[n * cols + k] + (int)zeros[n * G + j]);"),
    "dequant32_scale_transposed": ("out[n * cols + k] = d * scales[n * G + j];",
                                   "out[n * cols + k] = d * scales[j * rows + n];"),
    "dequant32_group_of_column": ("            int64_t j = k / group;\n            float d",
                                  "            int64_t j = k % G;\n            float d"),
    "dequant64_zero_sign": ("out[n * cols + k] = (double)((int)codes[n * cols + k] - (int)zeros[n * G + j])",
                            "out[n * cols + k] = (double)((int)codes[n * cols + k] + (int)zeros[n * G + j])"),
    "f16_scale_not_rounded": ("        s = bqo_f16_to_f32(bqo_f32_to_f16(s));\n", ""),
    "f16_round_half_away": ("    float n = nearbyintf(ldexpf(a, -ulp_exp));", "    float n = roundf(ldexpf(a, -ulp_exp));"),
    "f16_subnormal_step": ("    if (ulp_exp < -24) ulp_exp = -24;", "    if (ulp_exp < -25) ulp_exp = -25;"),
    "dequant64_scale_transposed": ("                                * (double)scales[n * G + j];\n        }\n}",
                                   "                                * (double)scales[j * rows + n];\n        }\n}"),
}

# cheap pins first; each mutant only has to fail one of them
PINS = [
    (P.test_worked_examples, {"name": "int4_g8_worked.txt"}),
    (P.test_worked_examples, {"name": "int2_g8_worked.txt"}),
    (P.test_worked_examples, {"name": "int4_clamp_worked.txt"}),
    (P.test_worked_examples, {"name": "int4_zero_tie_worked.txt"}),
    (P.test_page_scale_example, {}),
    (P.test_dequant_two_rows_two_groups, {}),
    (P.test_mixed_dequant_and_linear_tiled, {}),
    (P.test_constant_groups, {}),
    (P.test_interleaved_positions_hand_derived, {}),
    (P.test_meta_positions_hand_derived, {}),
    (P.test_decode_f16_all_patterns, {}),
    (P.test_invariants, {"bits": 4, "g": 32}),
    (P.test_linear_closed_form, {"bits": 4, "g": 128}),
    (P.test_brute_force_optimal_codes, {"bits": 2}),
    (P.test_exact_rational_arithmetic, {}),
    (P.test_sym_worked_examples, {"name": "sym_int4_g8_worked.txt"}),
    (P.test_sym_worked_examples, {"name": "sym_int2_g8_worked.txt"}),
    (P.test_sym_page_scale_example, {}),
    (P.test_grad_input_closed_form, {"bits": 4, "g": 128}),
    (P.test_grad_input_adjoint, {"bits": 4, "g": 32}),
    (P.test_f16_scale_worked_example, {}),
    (P.test_f32_to_f16_matches_library_rounding, {}),
    (P.test_f16_scale_exact_rational_arithmetic, {}),
]


def _build_mutant(tmp_path, name):
    src = open(os.path.join(os.path.dirname(O.__file__), "bq_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    c = tmp_path / f"{name}.c"
    c.write_text(src.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", *O.CFLAGS, str(c), "-o", str(so), "-lm"])
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    so = _build_mutant(tmp_path, name)
    caught = None
    with O.using_library(so):
        for fn, kw in PINS:
            try:
                fn(**kw)
            except (AssertionError, O.OracleError):
                caught = fn.__name__
                break
    assert caught is not None, f"mutant {name} passed every pin"


def test_unmutated_copy_passes(tmp_path):
    src = open(os.path.join(os.path.dirname(O.__file__), "bq_oracle.c")).read()
    c = tmp_path / "same.c"
    c.write_text(src)
    so = tmp_path / "same.so"
    subprocess.check_call(["gcc", *O.CFLAGS, str(c), "-o", str(so), "-lm"])
    with O.using_library(str(so)):
        for fn, kw in PINS:
            fn(**kw)
