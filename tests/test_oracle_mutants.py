"""Planted mistakes in the oracle: each plausible slip (a dropped term, a
wrong tie rule, a wrong rounding, a wrong code table, a wrong summation
order) is planted in a copy of the oracle's C source, built on the CPU, and
must make at least one pin in test_oracle_pins fail."""
import os
import subprocess

import pytest

import oracle
from oracle.build import CFLAGS
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "sbl_oracle.c")

MUTANTS = {
    "tie_rule_higher_index": ("float kj = fabsf(grp[j]);\n                    if (kj > ki || (kj == ki && j < i)) rank++;",
                              "float kj = fabsf(grp[j]);\n                    if (kj > ki || (kj == ki && j > i)) rank++;"),
    "round_half_away": ("float q = nearbyintf(r);", "float q = roundf(r);"),
    "sum_split_at_half": ("while (h * 2 < n) h *= 2;\n    double left = abs_sum_tree(w, lo, h);",
                          "h = n / 2;\n    double left = abs_sum_tree(w, lo, h);"),
    "gamma_over_dout_only": ("return (float)(s / (double)count);", "return (float)(s / (double)d_in);"),
    "act_divide_form": ("float s = bf16_to_f32(row[k]) * r;", "float s = bf16_to_f32(row[k]) / a * 127.0f;"),
    "act_scale_dropped": ("float v = nearbyintf(s);\n            if (v > 127.0f) v = 127.0f;\n            if (v < -128.0f) v = -128.0f;\n            q[t * d_in + k] = (int8_t)v;\n        }\n        d[t] = a / 127.0f;",
                          "float v = nearbyintf(s);\n            if (v > 127.0f) v = 127.0f;\n            if (v < -128.0f) v = -128.0f;\n            q[t * d_in + k] = (int8_t)v;\n        }\n        d[t] = a;"),
    "dequant_token_scale_dropped": ("float c = gamma * d[t];", "float c = gamma;"),
    "dw_token_scale_dropped": ("(double)bf16_to_f32(dy[t * d_out + o]) * (double)d[t] *\n                         (double)q[t * d_in + k];",
                               "(double)bf16_to_f32(dy[t * d_out + o]) *\n                         (double)q[t * d_in + k];"),
    "dx_gamma_dropped": ("dx[t * d_in + k] = (double)gamma * s;", "dx[t * d_in + k] = s;"),
    "mask_not_applied": ("weff[i] = (int8_t)(mask[i] ? wq[i] : 0);", "weff[i] = wq[i];"),
    "sign_extension_codes": ("return (uint8_t)(v + 1);", "return (uint8_t)(v & 3);"),
    "keep_rank_off_by_one": ("float kj = fabsf(grp[j]);\n                    if (kj > ki || (kj == ki && j < i)) rank++;\n                }\n                mask[o * d_in + g * m + i] = (uint8_t)(rank < n ? 1 : 0);",
                             "float kj = fabsf(grp[j]);\n                    if (kj > ki || (kj == ki && j < i)) rank++;\n                }\n                mask[o * d_in + g * m + i] = (uint8_t)(rank < n - 1 ? 1 : 0);"),
    "sp24_nibble_fields_swapped": ("unsigned nib = (unsigned)idx[0] | ((unsigned)idx[1] << 2);",
                                   "unsigned nib = (unsigned)idx[1] | ((unsigned)idx[0] << 2);"),
    "sp24_high_nibble_first": ("(nib << (4 * (g % 2)))", "(nib << (4 * (1 - g % 2)))"),
    "flips_count_agreements": ("if ((mask_prev[i] != 0) != (mask[i] != 0)) flips++;",
                               "if ((mask_prev[i] != 0) == (mask[i] != 0)) flips++;"),
    "near_zero_inclusive": ("if (r < 0.5f) c++;", "if (r <= 0.5f) c++;"),
    "threshold_from_kept": ("if (mask[k]) continue;\n                float a = fabsf(w[k]);",
                            "if (!mask[k]) continue;\n                float a = fabsf(w[k]);"),
    "survivor_gamma_over_all": ("return (float)(s / (double)kept);", "return (float)(s / (double)count);"),
    "quantized_mask_ties_high": ("int kj = grp[j] != 0;\n                    if (kj > ki || (kj == ki && j < i)) rank++;",
                                 "int kj = grp[j] != 0;\n                    if (kj > ki || (kj == ki && j > i)) rank++;"),
    "relu_not_squared": ("if (relu2) v = v > 0.0f ? v * v : 0.0f;", "if (relu2) v = v > 0.0f ? v : 0.0f;"),
    "residual_before_activation": ("if (relu2) v = v > 0.0f ? v * v : 0.0f;\n        if (res) v = v + bf16_to_f32(res[i]);",
                                   "if (res) v = v + bf16_to_f32(res[i]);\n        if (relu2) v = v > 0.0f ? v * v : 0.0f;"),
    "rmsnorm_eps_dropped": ("float r = (float)(1.0 / sqrt(s / (double)d_in + (double)eps));",
                            "float r = (float)(1.0 / sqrt(s / (double)d_in));"),
    "rmsnorm_mean_over_k_minus_1": ("float r = (float)(1.0 / sqrt(s / (double)d_in + (double)eps));",
                                    "float r = (float)(1.0 / sqrt(s / (double)(d_in - 1) + (double)eps));"),
    "rmsnorm_gain_ignored": ("            float u = bf16_to_f32(row[k]) * r;\n            if (g) u = u * bf16_to_f32(g[k]);\n            float v = nearbyintf(u * rq);",
                             "            float u = bf16_to_f32(row[k]) * r;\n            float v = nearbyintf(u * rq);"),
    "sp24_fill_from_top": ("for (int i = 0; i < 4 && count < 2; ++i) {\n                if (mask[o * d_in + 4 * g + i]) continue;",
                           "for (int i = 3; i >= 0 && count < 2; --i) {\n                if (mask[o * d_in + 4 * g + i]) continue;"),
    "t24_signs_swapped": ("(w[pos[0]] < 0 ? 2u : 0u) +\n                       (w[pos[1]] < 0 ? 1u : 0u);",
                          "(w[pos[0]] < 0 ? 1u : 0u) +\n                       (w[pos[1]] < 0 ? 2u : 0u);"),
    "t24_pair_table_order": ("{{-1, 0, 1, 2}, {-1, -1, 3, 4}, {-1, -1, -1, 5}",
                             "{{-1, 0, 1, 3}, {-1, -1, 2, 4}, {-1, -1, -1, 5}"),
    "t24_single_offset": ("code = 1u + 2u * (unsigned)pos[0] + (w[pos[0]] < 0 ? 1u : 0u);",
                          "code = 2u * (unsigned)pos[0] + (w[pos[0]] < 0 ? 1u : 0u);"),
    "ternarize_clip_dropped": ("if (q > 1.0f) q = 1.0f;\n        if (q < -1.0f) q = -1.0f;\n        wq[i] = (int8_t)q;",
                               "wq[i] = (int8_t)q;"),
    "pk2_codes_msb_first": ("int sh = (int)(2 * (k % 4));", "int sh = (int)(2 * (3 - k % 4));"),
    "pk2_padding_zero": ("for (int64_t b = 0; b < rb; ++b) row[b] = 0x55;", "for (int64_t b = 0; b < rb; ++b) row[b] = 0;"),
    "nm_bitmap_msb_first": ("brow[k / 8] = (uint8_t)(brow[k / 8] | (1u << (k % 8)));",
                            "brow[k / 8] = (uint8_t)(brow[k / 8] | (1u << (7 - k % 8)));"),
    "nm_values_msb_first": ("int sh = (int)(2 * (slot % 4));", "int sh = (int)(2 * (3 - slot % 4));"),
    "gemm_weights_transposed": ("s += (int64_t)q[t * d_in + k] * (int64_t)weff[o * d_in + k];",
                                "s += (int64_t)q[t * d_in + k] * (int64_t)weff[k * d_out + o];"),
    "acc_samples_token_for_row": ("acc += (int64_t)q[t * d_in + k] * (int64_t)weff[o * d_in + k];",
                                  "acc += (int64_t)q[o * d_in + k] * (int64_t)weff[t * d_in + k];"),
    "dx_samples_gamma_dropped": ("out[s] = (double)gamma * acc;", "out[s] = acc;"),
    "bf16_truncates": ("u += 0x7fffu + lsb;", "u += 0u * lsb;"),
    "dx_weights_transposed": ("s += (double)bf16_to_f32(dy[t * d_out + o]) * (double)weff[o * d_in + k];",
                              "s += (double)bf16_to_f32(dy[t * d_out + o]) * (double)weff[k * d_out + o];"),
    "dequant_accumulator_transposed": ("float v = (float)acc[t * d_out + o] * c;",
                                       "float v = (float)acc[o * tokens + t] * c;"),
    "t24_high_plane_stride": ("hrow[g / 4] = (uint8_t)(hrow[g / 4] | ((code >> 4) << (2 * (g % 4))));",
                              "hrow[g / 4] = (uint8_t)(hrow[g / 4] | ((code >> 4) << (2 * (g % 2))));"),
}

PIN_CALLS = [
    (pins.test_hand_row_6of8, ()),
    (pins.test_abs_sum_pairwise_order, ()),
    (pins.test_gamma_within_error_bound_of_exact_mean, ((128, 256),)),
    (pins.test_ternarize_ties_and_clip, ()),
    (pins.test_ternarize_matches_numpy_library_rounding, ()),
    (pins.test_mask_brute_force_tiny, (6, 8)),
    (pins.test_mask_degenerate_cases, ()),
    (pins.test_pk2_roundtrip_and_padding, ()),
    (pins.test_act_quant_invariants_and_zero_row, ()),
    (pins.test_act_quant_matches_numpy_float32, ()),
    (pins.test_output_matches_fp64_definition, ()),
    (pins.test_backward_matches_numpy_fp64, ()),
    (pins.test_nm_roundtrip, ()),
    (pins.test_sp24_hand_example, ()),
    (pins.test_sp24_roundtrip, (2, 4)),
    (pins.test_sp24_roundtrip, (1, 4)),
    (pins.test_t24_hand_row, ()),
    (pins.test_t24_all_groups, ()),
    (pins.test_t24_roundtrip, (2, 4)),
    (pins.test_epilogue_hand_values, ()),
    (pins.test_rmsnorm_quant_matches_numpy_definition, ()),
    (pins.test_gamma_survivors_hand_row_and_exact_mean, ()),
    (pins.test_mask_from_quantized_hand_and_brute_force, ()),
    (pins.test_mask_flips_matches_numpy_and_invariants, ()),
    (pins.test_near_zero_matches_numpy_and_gaussian_closed_form, ()),
    (pins.test_block_threshold_brute_force_and_hand_row, ()),
    (pins.test_gemm_acc_matches_numpy_int64, ()),
    (pins.test_gemm_acc_brute_force_tiny, ()),
    (pins.test_sampled_variants_agree_with_full, ()),
    (pins.test_epilogue_matches_numpy_float32_and_torch_bf16, ()),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", *CFLAGS, "-o", str(lib), str(mut), "-lm"], check=True)
    failed = []
    with oracle.use_library(str(lib)):
        for fn, args in PIN_CALLS:
            try:
                fn(*args)
            except (AssertionError, IndexError, ValueError):
                failed.append(fn.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
