"""Planted mistakes: each mutant copy of the oracle must fail at least one pin.

A mutant is the oracle's C++ source with one plausible error written into it
(a dropped term, a wrong index, a swapped operand, a wrong convention, a wrong rounding).  It is
compiled into a temporary library on the CPU, swapped in for the real one, and
the pins in test_oracle_pins are run against it.  Every mutant must be caught.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_fp8_pins as fp8
from tests import test_oracle_nvfp4_pins as fp4
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "beam_moe_oracle.cpp")

MUTANTS = {
    "group_score_is_max": ("gs[g] = per >= 2 ? v[0] + v[1] : v[0];", "gs[g] = v[0];"),
    "group_score_sums_all": ("gs[g] = per >= 2 ? v[0] + v[1] : v[0];",
                             "gs[g] = 0; for (float q : v) gs[g] += q;"),
    "bias_in_weights": ("static_cast<double>(S) * static_cast<double>(s[e]);",
                        "static_cast<double>(S) * static_cast<double>(sb[e]);"),
    "group_tie_upper_wins": ("      if (gs[a] != gs[b]) return gs[a] > gs[b];\n      return a < b;",
                             "      if (gs[a] != gs[b]) return gs[a] > gs[b];\n      return a > b;"),
    "expert_tie_upper_wins": ("      if (sb[a] != sb[b]) return sb[a] > sb[b];\n      return a < b;",
                              "      if (sb[a] != sb[b]) return sb[a] > sb[b];\n      return a > b;"),
    "select_by_unbiased_score": ("      if (sb[a] != sb[b]) return sb[a] > sb[b];",
                                 "      if (s[a] != s[b]) return s[a] > s[b];"),
    "down_proj_transposed": ("const uint16_t* wd = Wd + c * I;", "const uint16_t* wd = Wd + c;"),
    "no_silu": ("static_cast<double>(g) * sigmoid(static_cast<double>(g))",
                "static_cast<double>(g)"),
    "gate_up_swapped": ("static_cast<double>(g) * sigmoid(static_cast<double>(g))",
                        "static_cast<double>(u) * sigmoid(static_cast<double>(u))"),
    "no_normalisation": ("w[t * k + j] = static_cast<float>(norm_topk_prob ? num / denom : num);",
                         "w[t * k + j] = static_cast<float>(num);"),
    "residual_coefficient": ("const double cf = 1.0 / std::sqrt(kk);", "const double cf = 1.0 / kk;"),
    "rmsnorm_no_mean": ("std::sqrt(ss / static_cast<double>(d) + static_cast<double>(eps))",
                        "std::sqrt(ss + static_cast<double>(eps))"),
    "router_drops_last_term": ("      for (int64_t j = 0; j < d; ++j)\n        acc += static_cast<double>(bf16_bits_to_float(ht[j]))",
                               "      for (int64_t j = 0; j < d - 1; ++j)\n        acc += static_cast<double>(bf16_bits_to_float(ht[j]))"),
    "combine_drops_slot": ("      for (int j = 0; j < k; ++j)\n        acc += static_cast<double>(w[t * k + j])",
                           "      for (int j = 1; j < k; ++j)\n        acc += static_cast<double>(w[t * k + j])"),
    "bf16_truncates": ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;", ""),
    "bias_update_sign_flipped": ("const float sgn = c < mean ? 1.0f : (c > mean ? -1.0f : 0.0f);",
                                 "const float sgn = c < mean ? -1.0f : (c > mean ? 1.0f : 0.0f);"),
    "e4m3_truncates": ("double r = std::nearbyint(a / std::ldexp(1.0, E - 3));",
                       "double r = std::floor(a / std::ldexp(1.0, E - 3));"),
    "e4m3_subnormal_step": ("std::nearbyint(a / std::ldexp(1.0, -9))",
                            "std::nearbyint(a / std::ldexp(1.0, -10))"),
    "fp8_scale_divisor": ("const float s = amax / 448.0f;", "const float s = amax / 240.0f;"),
    "fp8_weight_scale_not_per_row": (
        "acc += xv[j] * value[w[j]];\n    y[c] = static_cast<float>(static_cast<double>(sx) * static_cast<double>(sw[c]) * acc",
        "acc += xv[j] * value[w[j]];\n    y[c] = static_cast<float>(static_cast<double>(sx) * static_cast<double>(sw[0]) * acc"),
    "fp8_down_reads_input_codes": ("linear_fp8_row(I, d, aq.data(), sa, Wdq, sd, y);",
                                   "linear_fp8_row(I, d, xq.data(), sx, Wdq, sd, y);"),
    "e2m1_truncates": ("mag = static_cast<uint8_t>(std::nearbyint(a / 0.5));",
                       "mag = static_cast<uint8_t>(std::floor(a / 0.5));"),
    "e2m1_middle_binade_step": ("mag = static_cast<uint8_t>(std::nearbyint(a) + 2.0);",
                                "mag = static_cast<uint8_t>(std::nearbyint(a / 2.0) * 2.0 + 2.0);"),
    "e2m1_exponent_bias": ("std::ldexp(1.0 + 0.5 * m, e - 1)", "std::ldexp(1.0 + 0.5 * m, e)"),
    "nvfp4_row_scale_divisor": ("const float s = amax / 2688.0f;", "const float s = amax / 448.0f;"),
    "nvfp4_block_scale_divisor": ("      t = t / 6.0f;", "      t = t / 4.0f;"),
    "nvfp4_block_max_is_row_max": ("    float mb = 0.0f;\n    for (int j = 0; j < 16; ++j) mb",
                                   "    float mb = amax;\n    for (int j = 0; j < 16; ++j) mb"),
    "nvfp4_linear_drops_input_block_scale": (
        "acc += e4m3_value(xbs[b]) * e4m3_value(wb[b]) * part;",
        "acc += e4m3_value(wb[b]) * part;"),
    "nvfp4_down_reads_input_codes": (
        "linear_nvfp4_row(I, d, aq.data(), ab.data(), sa, Wdq, Wdb, sd, y);",
        "linear_nvfp4_row(I, d, xq.data(), xb.data(), sx, Wdq, Wdb, sd, y);"),
}

PIN_TESTS = [
    (pins.test_route_matches_brute_force, [(8, 2, 1, 2), (16, 4, 2, 4)]),
    (pins.test_group_score_hand_examples, [()]),
    (pins.test_bias_is_selection_only, [()]),
    (pins.test_weights_sum_to_scaling_factor, [("tiny",)]),
    (pins.test_unnormalised_weights_are_scaled_scores, [()]),
    (pins.test_router_logits_match_float64_matmul, [()]),
    (pins.test_expert_mlp_matches_torch_float64, [()]),
    (pins.test_identical_experts_equal_scaled_dense_swiglu, [()]),
    (pins.test_combine_is_weighted_sum_of_expert_outputs, [()]),
    (pins.test_residual_coefficients_square_sum_is_one, [()]),
    (pins.test_residual_after_104_contributions_weighs_each_equally, [()]),
    (pins.test_rmsnorm_matches_torch_and_closed_form, [()]),
    (pins.test_bf16_rounding_matches_torch, [()]),
    (pins.test_bias_update_hand_example_and_invariants, [()]),
    (fp8.test_e4m3_decode_matches_torch_for_all_codes, [()]),
    (fp8.test_e4m3_encode_matches_torch_in_range_and_on_ties, [()]),
    (fp8.test_e4m3_saturates_and_keeps_nan, [()]),
    (fp8.test_quantize_rows_matches_torch_conversion_and_error_bounds, [()]),
    (fp8.test_quantize_rows_is_exact_on_representable_rows, [()]),
    (fp8.test_linear_fp8_equals_router_logits_on_exact_operands, [()]),
    (fp8.test_linear_fp8_general_scales_match_float64, [()]),
    (fp8.test_expert_mlp_fp8_gate_up_equal_bf16_expert_on_exact_operands, [()]),
    (fp8.test_expert_mlp_fp8_down_scales_are_per_output_row, [()]),
    (fp8.test_moe_tokens_fp8_is_weighted_sum_of_fp8_experts, [()]),
    (fp4.test_e2m1_decode_matches_the_format_table, [()]),
    (fp4.test_e2m1_encode_is_nearest_with_ties_to_even_and_saturates, [()]),
    (fp4.test_quantize_rows_nvfp4_is_exact_on_representable_rows, [()]),
    (fp4.test_quantize_rows_nvfp4_error_bounds_and_block_maxima, [()]),
    (fp4.test_quantize_rows_nvfp4_symmetries, [()]),
    (fp4.test_linear_nvfp4_matches_float64_on_decoded_operands, [()]),
    (fp4.test_linear_nvfp4_equals_router_logits_on_exact_operands, [()]),
    (fp4.test_expert_mlp_nvfp4_gate_up_equal_bf16_expert_on_exact_operands, [()]),
    (fp4.test_expert_mlp_nvfp4_down_uses_the_quantised_activation, [()]),
    (fp4.test_moe_tokens_nvfp4_is_weighted_sum_of_nvfp4_experts, [()]),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation {name} does not apply uniquely"
    path = tmp_path / f"{name}.cpp"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"lib{name}.so"
    subprocess.run(["g++", "-O1", "-std=c++17", "-ffp-contract=off", "-shared", "-fPIC",
                    "-pthread", "-o", str(so), str(path)], check=True)
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, monkeypatch, name):
    old, new = MUTANTS[name]
    so = _build_mutant(tmp_path, name, old, new)
    real = oracle.lib()
    mut = ctypes.CDLL(so)
    for fn in ("oracle_hardware_threads", "oracle_f32_to_bf16", "oracle_bf16_to_f32",
               "oracle_router_logits", "oracle_route", "oracle_expert_mlp", "oracle_moe_tokens",
               "oracle_rmsnorm", "oracle_residual", "oracle_residual_coefficients",
               "oracle_bias_update", "oracle_f32_to_e4m3", "oracle_e4m3_to_f32",
               "oracle_quantize_rows_e4m3", "oracle_linear_fp8", "oracle_expert_mlp_fp8",
               "oracle_moe_tokens_fp8", "oracle_f32_to_e2m1", "oracle_e2m1_to_f32",
               "oracle_quantize_rows_nvfp4", "oracle_linear_nvfp4", "oracle_expert_mlp_nvfp4",
               "oracle_moe_tokens_nvfp4"):
        f, g = getattr(real, fn), getattr(mut, fn)
        g.argtypes, g.restype = f.argtypes, f.restype
    monkeypatch.setattr(oracle, "_lib", mut)
    caught = []
    for test, params in PIN_TESTS:
        for p in params:
            try:
                test(*p)
            except (AssertionError, ValueError):
                caught.append(test.__name__)
                break
    assert caught, f"mutant {name} passed every pin"
