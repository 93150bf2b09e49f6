"""The pins must catch plausible mistakes in the oracle.

Each case copies fp8_oracle.c, plants one mistake (a wrong bias, a flipped
tie rule, a dropped term, a wrong sign, a transposed index), compiles the
copy on the CPU and runs the pins of tests/test_oracle_pins.py against it:
at least one pin must fail.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "fp8_oracle.c")

MUTATIONS = {
    "e4m3_bias": ("int bias = (fmt == ORC_E4M3) ? 7 : 15;", "int bias = (fmt == ORC_E4M3) ? 8 : 15;"),
    "subnormal_exponent": ("ldexp((double)Mt, 1 - bias - mbits)", "ldexp((double)Mt, -bias - mbits)"),
    "tie_to_odd": ("return (lo & 1u) ? hi : lo;", "return (lo & 1u) ? lo : hi;"),
    "f16_bias": ("ldexp((double)(1024 + Mt), E - 25)", "ldexp((double)(1024 + Mt), E - 24)"),
    "floor_at_tie": ("return (a <= f) ? (r - p) : (r - p - 1);", "return (a < f) ? (r - p) : (r - p - 1);"),
    "margin_sign": ("orc_fmt_max(fmt)) - margin;", "orc_fmt_max(fmt)) + margin;"),
    "mu_dropped": ("double t = mu * s_g;", "double t = s_g;"),
    "gemm_transposed_b": ("orc_fp8_decode(fb, B[j * b_sj + k * b_sk])", "orc_fp8_decode(fb, B[k * b_sj + j * b_sk])"),
    "gemm_descale_dropped": ("C[ij] = s * inv_sa * inv_sb", "C[ij] = s * inv_sa"),
    "adam_bias_correction_dropped": ("double mhat = m[i] / bc1;", "double mhat = m[i];"),
    "adam_sign": ("w[i] = w0[i] - lr * mhat", "w[i] = w0[i] + lr * mhat"),
    "adam_eps_inside_sqrt": ("(sqrt(vhat) + eps)", "sqrt(vhat + eps)"),
    "adam_beta2_swapped": ("v[i] = beta2 * v0[i] + (1.0 - beta2)", "v[i] = beta1 * v0[i] + (1.0 - beta1)"),
    "adam_wrong_scale_format": ("rc |= orc_compute_scale(am, ORC_E4M3, margin, s_m);",
                                "rc |= orc_compute_scale(am, ORC_F16, margin, s_m);"),
    "amax_nan_ignored": ("return saw_nan ? NAN : m;", "return m;"),
    "sharded_slice_amax_used": ("    if (amax_in) {", "    if (0 && amax_in) {"),
    "grad_scale_mu_dropped": ("    double t = mu * s;\n", "    double t = s;\n"),
    "sum_overflow_inclusive": ("        if (fabs(sum) > fmax)\n", "        if (fabs(sum) >= fmax)\n"),
    "cast_underflow_counts_zeros": ("if (!isnan(v) && v != 0.0 && code_value(fmt, c) == 0.0)",
                                    "if (!isnan(v) && code_value(fmt, c) == 0.0)"),
    "mu_quartered": ("*mu = (*mu * 0.5 < mu_min) ? mu_min : *mu * 0.5;",
                     "*mu = (*mu * 0.25 < mu_min) ? mu_min : *mu * 0.25;"),
    "mu_growth_late": ("    if (*clean >= interval) {", "    if (*clean > interval) {"),
    "sum_rounded_through_float": ("            sum += orc_fp8_decode(fmt, in[(size_t)r * ld + i]);",
                                  "            sum = (float)(sum + orc_fp8_decode(fmt, in[(size_t)r * ld + i]));"),
}

PINS = [
    pins.test_golden_format_points,
    lambda: pins.test_decode_table_matches_torch_float8(oracle.E4M3),
    lambda: pins.test_decode_table_matches_torch_float8(oracle.E5M2),
    lambda: pins.test_encode_brute_force_random_and_midpoints(oracle.E4M3),
    pins.test_f16_decode_matches_numpy_all_patterns,
    pins.test_f16_encode_matches_numpy,
    pins.test_amax_specials,
    pins.test_scale_closed_forms,
    pins.test_scale_invariants_and_mu,
    pins.test_cast_mu_invariance_codes_identical,
    lambda: pins.test_gemm_fwd_dgrad_wgrad_vs_numpy((3, 5, 7)),
    lambda: pins.test_adam_update_matches_torch_optim(2),
    pins.test_adam_step_composition_with_independent_pieces,
    pins.test_adam_sharded_equals_whole_tensor_step,
    lambda: pins.test_cast_counts_closed_forms(oracle.E5M2),
    pins.test_grad_scale_closed_forms,
    lambda: pins.test_sum_codes_vs_torch(oracle.E5M2, 3),
    pins.test_sum_codes_specials,
    pins.test_mu_update_hand_traced,
    pins.test_fp8_allreduce_pre_post_auto_hand_built,
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(mutated),
                           "-o", str(lib), "-lm"])
    failures = 0
    with oracle.use_library(str(lib)):
        for pin in PINS:
            try:
                pin()
            except AssertionError:
                failures += 1
    assert failures >= 1, f"no pin caught mutation {name}"
