"""The oracle's pins are sensitive: a copy of the oracle with one planted
mistake (compiled on the CPU into a temporary directory, never committed)
must fail at least one pin.  Each mutation is a plausible slip: a wrong tie
rule, a wrong qmax, a signed max in place of the absmax, a dropped term, a
transposed index, a wrong group index.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
import tests.test_oracle_ext_pins as ext
import tests.test_oracle_lowrank_pins as lr
import tests.test_oracle_nvfp4_pins as nv
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "wlq_oracle.c")

MUTATIONS = {
    "ties_round_up": ("return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "return f + 1.0;"),
    "qmax_off_by_one": ("const double qmax = (double)((1 << (bits - 1)) - 1);",
                        "const double qmax = (double)(1 << (bits - 1));"),
    "bias_dropped": ("if (bias) acc += bf16_value(bias[n]);", "(void)bias;"),
    "low_rank_transposed": ("acc += T[j] * bf16_value(L2[(int64_t)j * N + n]);",
                            "acc += T[j] * bf16_value(L2[n * (int64_t)r + j]);"),
    "group_index": ("(double)scales[n * G + k / g];\n                acc",
                    "(double)scales[n * G + k % G];\n                acc"),
    "signed_max": ("double v = fabs((double)w[k]);", "double v = (double)w[k];"),
    "format_rounds_down": ("const double r = round_half_even(x / spacing) * spacing;",
                           "const double r = floor(x / spacing) * spacing;"),
    "sixteen_bit_scale_kept_fp32": ("if (scale_dtype == 0) s = (double)(float)qd;",
                                    "if (scale_dtype >= 0) s = (double)(float)qd;"),
    "fp8_max_off": ("const float s = (float)(a / 448.0);", "const float s = (float)(a / 480.0);"),
    "residual_l1_transposed": ("bf16_value(L1[k * r + j]) * bf16_value(L2[(int64_t)j * N + n]);",
                               "bf16_value(L1[(int64_t)j * K + k]) * bf16_value(L2[(int64_t)j * N + n]);"),
    "residual_last_rank_dropped": ("for (int j = 0; j < r; ++j) {\n                const double prod",
                                   "for (int j = 0; j < r - 1; ++j) {\n                const double prod"),
    "residual_sign": ("const double d = (double)W[n * K + k] - p;", "const double d = (double)W[n * K + k] + p;"),
    "nvfp4_tensor_scale_off": ("(float)(amax / (6.0 * 448.0))", "(float)(amax / (6.0 * 480.0))"),
    "nvfp4_block_max_signed": ("const double v = fabs(in_value(X, x_dtype, base + j));",
                               "const double v = in_value(X, x_dtype, base + j);"),
    "e2m1_no_subnormals": ("round_to_format(fabs(t), 2, 0, 6.0)", "round_to_format(fabs(t), 2, 1, 6.0)"),
    "e2m1_sign_dropped": ("return (uint8_t)(code | (neg << 3));", "(void)neg; return code;"),
    "nvfp4_weight_block_index": ("e4m3_value(ws[n * (K / 16) + k / 16])", "e4m3_value(ws[n * (K / 16) + k % (K / 16)])"),
    "nvfp4_low_rank_dropped": ("y[m * N + n] = acc + lr + b;", "y[m * N + n] = acc + b;"),
    "nvfp4_e4m3_decode_bias": ("ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
}

PIN_TESTS = [
    lambda: pins.test_quantize_matches_brute_force(8),
    lambda: pins.test_quantize_matches_brute_force(4),
    lambda: pins.test_exact_ties_round_to_even(),
    lambda: pins.test_grouping_matches_brute_force(4, 16),
    lambda: pins.test_rtn_error_bound(4, 64),
    lambda: pins.test_linear_exact_rationals_tiny(),
    lambda: pins.test_linear_matches_numpy_matmul(4, 16),
    lambda: pins.test_linear_matches_numpy_matmul(8, 0),
    lambda: pins.test_linear_low_rank_only_and_plain_only(),
    lambda: ext.test_codes_are_the_brute_force_nearest_with_the_stored_scale(5, oracle.SCALE_F16),
    lambda: ext.test_codes_are_the_brute_force_nearest_with_the_stored_scale(3, oracle.SCALE_BF16),
    lambda: ext.test_fp8_codes_are_the_nearest_e4m3_ties_to_even_saturated(),
    lambda: ext.test_fp8_codes_match_torch_e4m3fn_conversion(),
    lambda: lr.test_residual_equals_fp64_matmul_when_every_sum_is_exact(),
    lambda: nv.test_every_e2m1_code_and_midpoint_with_unit_scales(),
    lambda: nv.test_block_scales_are_the_nearest_e4m3_with_ties_to_even(),
    lambda: nv.test_codes_are_the_brute_force_nearest_for_random_tensors(),
    lambda: nv.test_dequantize_decodes_the_fields(),
    lambda: nv.test_w4a4_linear_matches_numpy_matmul(16, True),
    lambda: nv.test_w4a4_linear_exact_small_case(),
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "mut.c")
        so = os.path.join(d, "libmut.so")
        open(c, "w").write(src.replace(old, new))
        subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-shared", "-fPIC", c, "-o", so, "-lm"])
        monkeypatch.setattr(oracle, "_lib", oracle.bind(so))
        failures = 0
        for t in PIN_TESTS:
            try:
                t()
            except (AssertionError, oracle.OracleError):
                failures += 1
        assert failures > 0, "mutation %s slipped past every pin" % name
