"""Planted mistakes in a copy of the oracle must each fail some pin (CPU only).

Every mutant is a one-place textual change to a temporary copy of
``oracle/oracle.c`` -- a dropped term, a wrong comparison, a wrong index,
a wrong rounding -- compiled into its own library.  The committed oracle
is never modified.  If a mutant passed every pin, the pins would not be
pinning the oracle down.
"""
import os
import shutil
import subprocess

import pytest

import oracle
import oracle_pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "drop_16bit_part": ("+ y16[n];", "+ 0.0;"),
    "outlier_rule_strict": (">= alpha)\n                is_outlier[k] = 1;", "> alpha)\n                is_outlier[k] = 1;"),
    "row_scale_includes_outliers": ("if (is_outlier[k]) continue;", "(void)0;"),
    "outlier_code_not_zeroed": ("is_outlier[k] ? 0 : quantise_one", "is_outlier[k] ? quantise_one(orc_half_to_float(xrow[k]), inv) : quantise_one"),
    "dequant_by_127_not_127sq": ("/ 16129.0", "/ 127.0"),
    "round_half_even": ("if (fabsf(v - r) >= 0.5f) r += copysignf(1.0f, v);", "r = nearbyintf(v);"),
    "round_half_up_strict": ("if (fabsf(v - r) >= 0.5f)", "if (fabsf(v - r) > 0.5f)"),
    "weight_scale_per_row": ("float a = fabsf(orc_half_to_float(W16[(size_t)k * N + n]));",
                             "float a = fabsf(orc_half_to_float(W16[(size_t)(n % K) * N + (k % N)]));"),
    "gemm_transposed_weight": ("const int8_t *wrow = Wq + (size_t)k * N;", "const int8_t *wrow = Wq + (size_t)(k % N) * N;"),
    "outlier_w_row_index": ("wrow = W16 + (size_t)k * N;", "wrow = W16 + (size_t)j * N;"),
    "dequant_scale_128": ("float d = sW[n] / 127.0f;", "float d = sW[n] / 128.0f;"),
    "dequant_biased": ("float v = (float)Wq[(size_t)k * N + n] * d;", "float v = (float)Wq[(size_t)k * N + n] * d * 0.999f;"),
    "wq_variant_row_index": ("orc_dequantize_weight(Wq + (size_t)k * N, sW, 1, N, wdq);",
                             "orc_dequantize_weight(Wq + (size_t)j * N, sW, 1, N, wdq);"),
    "half_subnormal_exponent": ("mag = ldexp((double)frac, -24);", "mag = ldexp((double)frac, -25);"),
    "y_round_truncate": ("if (diff > 0.5) return fl + 1.0;", "if (diff > 2.0) return fl + 1.0;"),
    "scale_x_instead_of_w": ("* (double)sX[r] * (double)sW[n]", "* (double)sX[r] * (double)sX[r]"),
    "reciprocal_two_roundings": ("float v = x * inv;", "float v = (x * 127.0f) / (127.0f / inv);"),
    # the group-wise 4-bit codec
    "int4_step_by_16": ("(range / 15.0f)", "(range / 16.0f)"),
    "int4_code_truncates": ("float r = orc_rhaz(d * inv);", "float r = truncf(d * inv);"),
    "int4_group_skips_first_row": ("for (int k = g * G; k < (g + 1) * G; ++k) {\n                float w",
                                   "for (int k = g * G + 1; k < (g + 1) * G; ++k) {\n                float w"),
    "int4_codes_from_zero_not_lo": ("W16[(size_t)k * N + n]) - lo;", "W16[(size_t)k * N + n]) - 0.0f;"),
    "int4_decode_drops_lo": ("+ (double)orc_half_to_float(lo[gi]);", "+ 0.0;"),
    "int4_product_wrong_row": ("const uint16_t *wrow = Wd + (size_t)k * N;",
                               "const uint16_t *wrow = Wd + (size_t)(k ^ 1) * N;"),
    # sign and extremum slips
    "outlier_test_signed": ("if (fabsf(orc_half_to_float(X[(size_t)t * K + k])) >= alpha)\n                is_outlier[k] = 1;",
                            "if (orc_half_to_float(X[(size_t)t * K + k]) >= alpha)\n                is_outlier[k] = 1;"),
    "row_scale_signed_max": ("float a = fabsf(orc_half_to_float(xrow[k]));", "float a = orc_half_to_float(xrow[k]);"),
    "int4_lo_first_not_min": ("if (w < lo) lo = w;", "if (k == g * G) lo = w;"),
    # the 4-bit codec's rounding steps
    "int4_code_ties_to_even": ("float r = orc_rhaz(d * inv);", "float r = nearbyintf(d * inv);"),
    "int4_codes_from_unrounded_step": ("float s = orc_half_to_float(s16);", "float s = range / 15.0f;"),
    "int4_decode_two_roundings": ("double v = (double)codes[(size_t)k * N + n] * (double)orc_half_to_float(scale[gi])",
                                  "double v = (double)orc_half_to_float(orc_double_to_half((double)codes[(size_t)k * N + n]"
                                  " * (double)orc_half_to_float(scale[gi])))"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/not found"
    d = tmp_path / name
    d.mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "oracle.h"), d / "oracle.h")
    (d / "oracle.c").write_text(src.replace(old, new))
    so = d / "liboracle_mutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
                    "-shared", "-fPIC", str(d / "oracle.c"), "-o", str(so), "-lm"], check=True)
    mutant = oracle.Oracle(oracle.lib(str(so)))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ArithmeticError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
