"""Pin strength: plant plausible mistakes in copies of the oracle source and
check that the pins catch every one.  The mistakes live only in temporary
copies compiled on the CPU; the committed oracle is never changed."""
from __future__ import annotations

import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

MUTATIONS = {
    "threshold_strict": ("if (fabsf(x) >= thr)", "if (fabsf(x) > thr)"),
    "outliers_in_row_absmax": ("if (is_out[k]) continue;", ";"),
    "outlier_column_not_zeroed": ("if (!is_out[k] && amax > 0.0f)", "if (amax > 0.0f)"),
    "round_half_away": ("float r = nearbyintf(x * scale);", "float r = roundf(x * scale);"),
    "divide_instead_of_scale": ("float r = nearbyintf(x * scale);", "float r = nearbyintf(x / (1.0f / scale));"),
    "clamp_to_126": ("if (r > 127.0f) r = 127.0f;", "if (r > 126.0f) r = 126.0f;"),
    "weight_transposed": ("float a = fabsf(orc_half_to_float(W[(size_t)k * N + n]));",
                          "float a = fabsf(orc_half_to_float(W[(size_t)(k % N) * N + (n % K)]));"),
    "weight_absmax_skips_row0": ("for (int k = 0; k < K; ++k) {\n            float a = fabsf(orc_half_to_float(W[",
                                 "for (int k = 1; k < K; ++k) {\n            float a = fabsf(orc_half_to_float(W["),
    "gemm_drops_last_k": ("for (int k = 0; k < j->K; ++k) s +=", "for (int k = 0; k + 1 < j->K; ++k) s +="),
    "outlier_term_dropped": ("v = v + o;", "v = v + 0.0f * o;"),
    "outlier_sign": ("v = v + o;", "v = v - o;"),
    "wrong_denominator": ("v = v / 16129.0f;", "v = v / 16384.0f;"),
    "kept_row_ignored": ("if (slot >= 0) {\n                w = W_keep", "if (slot >= 1000000) {\n                w = W_keep"),
    "xo_wrong_column": ("Xo[(size_t)m * n_o + j] = row[idx[j]];", "Xo[(size_t)m * n_o + j] = row[idx[j] > 0 ? idx[j] - 1 : 0];"),
    "threshold_signed": ("if (fabsf(x) >= thr)", "if (x >= thr)"),
    "detect_first_row_only": ("for (int m = 0; m < M; ++m) {\n            float x = orc_half_to_float(X[",
                              "for (int m = 0; m < 1; ++m) {\n            float x = orc_half_to_float(X["),
    "outlier_list_descending": ("for (int k = 0; k < K; ++k) {\n        int flag = 0;",
                                "for (int k = K - 1; k >= 0; --k) {\n        int flag = 0;"),
    "row_absmax_signed": ("float a = fabsf(orc_half_to_float(row[k]));", "float a = orc_half_to_float(row[k]);"),
    "weight_absmax_signed": ("float a = fabsf(orc_half_to_float(W[(size_t)k * N + n]));",
                             "float a = orc_half_to_float(W[(size_t)k * N + n]);"),
    "product_in_double": ("float r = nearbyintf(x * scale);", "float r = (float)nearbyint((double)x * (double)scale);"),
    "epilogue_ra_twice": ("v = v * ca;", "v = v * ra;"),
    "dequantised_row_over_128": ("w = orc_float_to_half(t / 127.0f);", "w = orc_float_to_half(t / 128.0f);"),
    "outlier_weight_rows_reversed": ("orc_half_to_float(Wo[(size_t)j * N + n]);",
                                     "orc_half_to_float(Wo[(size_t)(n_o - 1 - j) * N + n]);"),
    "half_subnormal_exponent": ("v = ldexpf((float)mant, -24);", "v = ldexpf((float)mant, -25);"),
    "half_encode_truncates": ("float m = nearbyintf(ldexpf(a, 10 - e));", "float m = truncf(ldexpf(a, 10 - e));"),
}

# mistakes in the variants (block-wise codec, group-wise matmul, 4-bit product)
VARIANT_MUTATIONS = {
    "block_short_by_one": ("long hi = lo + B < n ? lo + B : n;", "long hi = lo + B - 1 < n ? lo + B - 1 : n;"),
    "block_absmax_whole_vector": ("for (long i = lo; i < hi; ++i) {\n            float a = fabsf(x[i]);",
                                  "for (long i = 0; i < n; ++i) {\n            float a = fabsf(x[i]);"),
    "block_dequant_over_128": ("out[i] = t / 127.0f;", "out[i] = t / 128.0f;"),
    "block_dequant_next_constant": ("float t = (float)q[i] * absmax[i / B];",
                                    "float t = (float)q[i] * absmax[(i + 1) / B < (n + B - 1) / B ? (i + 1) / B : i / B];"),
    "grouped_x_absmax_whole_row": ("for (int k = g * G; k < (g + 1) * G; ++k) {\n                if (is_out[k]) continue;",
                                   "for (int k = 0; k < K; ++k) {\n                if (is_out[k]) continue;"),
    "grouped_outliers_in_absmax": ("                if (is_out[k]) continue;\n                float a", "                float a"),
    "grouped_w_absmax_whole_column": (
        "for (int k = g * G; k < (g + 1) * G; ++k) {\n                float a = fabsf(orc_half_to_float(W[(size_t)k * N + n]));"
        "\n                if (a > amax) amax = a;\n            }\n            ca[(size_t)n * ng + g] = amax;\n"
        "            float scale = amax > 0.0f ? 127.0f",
        "for (int k = 0; k < K; ++k) {\n                float a = fabsf(orc_half_to_float(W[(size_t)k * N + n]));"
        "\n                if (a > amax) amax = a;\n            }\n            ca[(size_t)n * ng + g] = amax;\n"
        "            float scale = amax > 0.0f ? 127.0f"),
    "grouped_epilogue_first_constant": ("t = t * ca[(size_t)n * ng + g];", "t = t * ca[(size_t)n * ng];"),
    "grouped_sum_drops_last_group": ("v = v + t;\n            }", "if (g + 1 < ng || ng == 1) v = v + t;\n            }"),
    "grouped_dequant_row_first_constant": ("Wq[(size_t)n * K + k] * ca[(size_t)n * ng + k / G]",
                                           "Wq[(size_t)n * K + k] * ca[(size_t)n * ng]"),
    "int4_clamp_at_6": ("if (r > 7.0f) r = 7.0f;", "if (r > 6.0f) r = 6.0f;"),
    "int4_scale_over_8": ("float scale = amax > 0.0f ? 7.0f / amax : 0.0f;", "float scale = amax > 0.0f ? 8.0f / amax : 0.0f;"),
    "int4_dequant_over_8": ("float w = t / 7.0f;\n                s += (double)orc_half_to_float(X[(size_t)m * K + k])",
                            "float w = t / 8.0f;\n                s += (double)orc_half_to_float(X[(size_t)m * K + k])"),
    "int4_dequant_first_group": ("ca[(size_t)n * ng + k / G];\n                float w", "ca[(size_t)n * ng];\n                float w"),
    "int4_sum_through_fp32": ("Y[(size_t)m * N + n] = orc_double_to_half(s);", "Y[(size_t)m * N + n] = orc_float_to_half((float)s);"),
    "int4_half_round_truncates": ("double m = nearbyint(ldexp(a, 10 - e));", "double m = trunc(ldexp(a, 10 - e));"),
}


def _run(checks, first_only=False):
    """Run the checks in order; return the names of those that fail (only the
    first one when first_only: a planted mistake is caught by any pin)."""
    failed = []
    for name, fn in checks.items():
        try:
            fn()
        except Exception:  # noqa: BLE001 - any failure counts as caught
            failed.append(name)
            if first_only:
                break
    return failed


def _variant_pin_suite(first_only=False):
    """A fast subset of the variants' pins; return the names of those that fail."""
    from tests import test_oracle_variant_pins as vp

    checks = {
        "block_golden": vp.test_block_worked_example_golden,
        "block_isolation": vp.test_block_outlier_stays_in_its_block,
        "block_integers": vp.test_block_integers_round_trip_exactly,
        "grouped_one_group": lambda: vp.test_grouped_with_one_group_is_the_vectorwise_method(False),
        "grouped_integers": vp.test_grouped_integer_inputs_give_the_exact_product,
        "grouped_error_bound": vp.test_grouped_result_within_method_error_bound,
        "double_to_half": vp.test_double_to_half_rounds_once,
        "int4_single_rounding": vp.test_int4_rounds_the_sum_once,
        "int4_bound": vp.test_int4_absmax_maps_to_7_and_error_within_half_step,
        "int4_integers": vp.test_int4_integer_weights_are_exact,
    }
    for seed in range(30):
        checks[f"block_brute_force_{seed}"] = (lambda s=seed: vp.test_block_brute_force(s))
        checks[f"grouped_brute_force_{seed}"] = (lambda s=seed: vp.test_grouped_brute_force_tiny(s))
        checks[f"int4_brute_force_{seed}"] = (lambda s=seed: vp.test_int4_brute_force_tiny(s))
    return _run(checks, first_only)


def _pin_suite(first_only=False):
    """Run a fast subset of the pins, cheapest first; return the names of
    those that fail."""
    checks = {
        "worked_example": pins.test_worked_example_golden,
        "threshold_equality": pins.test_value_exactly_at_threshold_is_outlier,
        "absmax_127": pins.test_absmax_maps_to_127,
        "lossless": pins.test_lossless_integer_inputs,
        "all_outlier": pins.test_all_outlier_reduces_to_fp16_matmul,
        "error_bound": pins.test_result_within_method_error_bound,
        "dequantised_rows": pins.test_dequantised_outlier_rows_when_not_kept,
    }
    for seed in range(40):
        checks[f"brute_force_{seed}"] = (lambda s=seed: pins.test_brute_force_tiny(s))
    checks["half_decode"] = pins.test_half_to_float_exhaustive
    checks["half_encode"] = pins.test_float_to_half_round_half_even
    for amax in (5.99609375, 3.140625, 40.96875, 0.46044921875, 1.5947265625):
        checks[f"rule_exhaustive_{amax}"] = (lambda a=amax: pins.test_quantisation_rule_exhaustive(a))
    return _run(checks, first_only)


VARIANTS_MARKER = "Variants beyond the vector-wise matmul"


def _mutated_suite_failures(old, new, suite, tmp_path, variant):
    """Plant the mistake at the anchor's first occurrence, which must lie in
    the vector-wise part of the source (or, for a variant, be the only one and
    lie in the variants' part); return the pins that fail."""
    with open(oracle._SRC) as f:
        src = f.read()
    at, marker = src.find(old), src.find(VARIANTS_MARKER)
    assert at >= 0 and marker >= 0, f"mutation anchor {old!r} not found"
    if variant:
        assert at > marker and src.count(old) == 1, f"variant anchor {old!r} must occur once, among the variants"
    else:
        assert at < marker, f"anchor {old!r} must first occur in the vector-wise part"
    mutated = src.replace(old, new, 1)
    c_path = os.path.join(tmp_path, "mut.c")
    so_path = os.path.join(tmp_path, "libmut.so")
    with open(c_path, "w") as f:
        f.write(mutated)
    subprocess.run(["gcc", *oracle._CFLAGS, "-o", so_path, c_path, "-lm"], check=True)
    oracle._swap_library(so_path)
    try:
        return suite()
    finally:
        oracle._swap_library(None)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    suite = lambda: _pin_suite(first_only=True)  # noqa: E731
    assert _mutated_suite_failures(old, new, suite, tmp_path, False), f"planted mistake {name!r} passed every pin"


@pytest.mark.parametrize("name", sorted(VARIANT_MUTATIONS))
def test_planted_variant_mistake_is_caught(name, tmp_path):
    old, new = VARIANT_MUTATIONS[name]
    suite = lambda: _variant_pin_suite(first_only=True)  # noqa: E731
    assert _mutated_suite_failures(old, new, suite, tmp_path, True), f"planted mistake {name!r} passed every pin"


def test_unmutated_oracle_passes_suite():
    assert _pin_suite() == []
    assert _variant_pin_suite() == []
