"""Planted-mistake checks for the oracle's pins (CPU only).

Each case copies attention_ref.c, plants one plausible mistake (a transposed
operand, a wrong head map, a dropped scale, an off-by-one mask, a wrong log
base, a wrong exponent bias, the wrong rounding rule; in the backward a
dropped delta term, a wrong operand, a missing head of the group), builds the copy with
gcc and runs the pins against it: at least one pin must fail.  The planted
copies live in a temporary directory; the committed oracle is untouched."""
import os

import pytest

import oracle
import tests.test_oracle_bwd_pins as bwd_pins
import tests.test_oracle_fp8_pins as fp8_pins
import tests.test_oracle_mask_pins as mask_pins
import tests.test_oracle_pins as pins
from exact_attention_113_b200.inputs import F16, BF16

SRC = os.path.join(os.path.dirname(oracle.__file__), "attention_ref.c")

MUTATIONS = {
    "k_transposed": ("acc += qrow[d] * tab[kp[j * D + d]];",
                     "acc += qrow[d] * tab[kp[d * L_k + j]];"),
    "v_reads_k": ("o[d] += p[j] * tab[vp[j * D + d]];",
                  "o[d] += p[j] * tab[kp[j * D + d]];"),
    "gqa_modulo": ("int64_t g = h / group;                       /* GQA head map */",
                   "int64_t g = h % H_kv;"),
    "scale_dropped": ("\n                s[j] = scale * acc;", "\n                s[j] = acc;"),
    "window_off_by_one": ("if (wl >= 0 && j < i - wl) return 0;",
                          "if (wl >= 0 && j <= i - wl) return 0;"),
    "causal_off_by_one": ("if (causal && j > i) return 0;",
                          "if (causal && j >= i) return 0;"),
    "lse_log2": ("lse[t] = (m == -INFINITY) ? -INFINITY : m + log(den);",
                 "lse[t] = (m == -INFINITY) ? -INFINITY : m + log2(den);"),
    "f16_bias": ("v = ldexp((double)(1024 + m), e - 25);",
                 "v = ldexp((double)(1024 + m), e - 24);"),
    "bf16_bias": ("v = ldexp((double)(128 + m), e - 134);",
                  "v = ldexp((double)(128 + m), e - 133);"),
    "round_half_away": ("double r = nearbyint(ldexp(a, -q_exp));",
                        "double r = round(ldexp(a, -q_exp));"),
    "wabs_signed": ("w[d] += p[j] * fabs(tab[vp[j * D + d]]);",
                    "w[d] += p[j] * tab[vp[j * D + d]];"),
    "wrss_no_root": ("                    w[d] = sqrt(w[d]);", "                    w[d] = w[d];"),
    "wrss_weight_not_squared": ("const double term = p[j] * tab[vp[j * D + d]];\n                        w[d] += term * term;",
                                "const double term = tab[vp[j * D + d]];\n                        w[d] += p[j] * term * term;"),
    "online_stale_max": ("d = d * exp(m - m_new) + exp(x[i] - m_new);",
                         "d = d + exp(x[i] - m_new);"),
    # backward
    "bwd_delta_dropped": ("ds[j] = p[j] * (dp[j] - delta);", "ds[j] = p[j] * dp[j];"),
    "bwd_dk_reads_k": ("dkp[j * D + d] += scale * ds[j] * qi[d];",
                       "dkp[j * D + d] += scale * ds[j] * kp[j * D + d];"),
    "bwd_dq_scale_dropped": ("dqi[d] += scale * ds[j] * kp[j * D + d];",
                             "dqi[d] += ds[j] * kp[j * D + d];"),
    "bwd_dv_uses_ds": ("dvp[j * D + d] += p[j] * doi[d];", "dvp[j * D + d] += ds[j] * doi[d];"),
    "bwd_dp_reads_k": ("if (p[j] != 0.0)\n                            for (int64_t d = 0; d < D; d++) acc += doi[d] * vp[j * D + d];",
                       "if (p[j] != 0.0)\n                            for (int64_t d = 0; d < D; d++) acc += doi[d] * kp[j * D + d];"),
    "bwd_group_last_head_only": ("for (int64_t h = g * group; h < (g + 1) * group; h++)",
                                 "for (int64_t h = (g + 1) * group - 1; h < (g + 1) * group; h++)"),
    "bwd_abs_signed": ("if (dva) dva[j * D + d] += p[j] * fabs(doi[d]);",
                       "if (dva) dva[j * D + d] += p[j] * doi[d];"),
    "bwd_abs_delta_term_dropped": ("const double wabs_j = fabs(ds[j]) + p[j] * e;",
                                   "const double wabs_j = fabs(ds[j]);"),
    # fp8
    "e4m3_bias": ("v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 9);"),
    "e4m3_subnormal_scale": ("v = ldexp((double)m, -9);                /* subnormal: m * 2^-9 */",
                             "v = ldexp((double)m, -10);"),
    "e4m3_nan_missed": ("if (e == 0xf && m == 0x7)", "if (e == 0xf && m == 0x8)"),
    "bwd_mask_bias_dropped": ("s[j] = scale * acc + bias;", "s[j] = scale * acc;"),
    "bwd_mask_row_stride_ignored": ("h * stride_h +\n                                                                   i * stride_q + j, &hidden);",
                                    "h * stride_h +\n                                                                   j, &hidden);"),
    # mask and statistics
    "mask_bool_inverted": ("*hidden = ((const uint8_t *)mask)[idx] != 0;",
                           "*hidden = ((const uint8_t *)mask)[idx] == 0;"),
    "mask_bias_dropped": ("s[j] += bias;", "s[j] += 0.0;"),
    "mask_row_stride_ignored": ("b * stride_b + h * stride_h + i * stride_q + j",
                                "b * stride_b + h * stride_h + j"),
    "ssum_not_relative_to_max": ("if (ssum) ssum[t] = (m == -INFINITY) ? 0.0 : den;",
                                 "if (ssum) ssum[t] = (m == -INFINITY) ? 0.0 : den * exp(m);"),
    "f64_forward_wrong_head": ("const double *kp = k + (b * H_kv + h / group) * L_k * D;\n            const double *vp",
                               "const double *kp = k + (b * H_kv + h % H_kv) * L_k * D;\n            const double *vp"),
}


def _battery(orc):
    """Every pin, called on the given oracle build."""
    yield lambda: pins.test_decode_matches_library_on_every_pattern(orc, F16)
    yield lambda: pins.test_decode_matches_library_on_every_pattern(orc, BF16)
    yield lambda: pins.test_round_f16_matches_numpy(orc)
    yield lambda: pins.test_round_bf16_matches_torch(orc)
    yield lambda: pins.test_online_softmax_worked_example(orc)
    yield lambda: pins.test_online_equals_three_pass_random(orc)
    for case in pins.BRUTE_CASES:
        yield lambda case=case: pins.test_matches_brute_force(orc, case)
    for c in (False, True):
        yield lambda c=c: pins.test_matches_torch_fp64_softmax(orc, c)
    yield lambda: pins.test_causal_row_zero_is_v0(orc)
    yield lambda: pins.test_zero_keys_give_mean_of_visible_values(orc, True, 4)
    yield lambda: pins.test_gqa_equals_mha_with_repeated_heads(orc)
    yield lambda: pins.test_shifting_every_key(orc)
    yield lambda: pins.test_fully_masked_rows(orc)
    yield lambda: pins.test_weighted_abs_value_closed_forms(orc)
    yield lambda: pins.test_weighted_rss_closed_forms(orc)
    for c in bwd_pins.CASES:
        yield lambda c=c: bwd_pins.test_finite_differences_of_the_forward(orc, c)
        yield lambda c=c: bwd_pins.test_matches_torch_fp64_autograd(orc, c)
    yield lambda: bwd_pins.test_single_key(orc)
    yield lambda: bwd_pins.test_scale_zero(orc)
    yield lambda: bwd_pins.test_constant_values(orc)
    yield lambda: bwd_pins.test_gqa_gradient_sums_the_group(orc)
    yield lambda: bwd_pins.test_linear_in_dout(orc)
    for dt in (F16, BF16):
        yield lambda dt=dt: bwd_pins.test_bit_pattern_entry_decodes_exactly(orc, dt)
    yield lambda: bwd_pins.test_error_scales(orc)
    yield lambda: bwd_pins.test_masked_backward_finite_differences(orc)
    yield lambda: bwd_pins.test_masked_backward_matches_torch_autograd(orc)
    yield lambda: bwd_pins.test_causal_pattern_mask_equals_causal_backward(orc)
    yield lambda: fp8_pins.test_decode_every_code_matches_torch(orc)
    yield lambda: fp8_pins.test_decode_closed_points(orc)
    yield lambda: fp8_pins.test_attention_on_e4m3_equals_fp16_of_same_values(orc)
    yield lambda: mask_pins.test_empty_masks_change_nothing(orc)
    yield lambda: mask_pins.test_causal_pattern_masks(orc)
    yield lambda: mask_pins.test_row_constant_shift(orc)
    yield lambda: mask_pins.test_log_weight_mask_reweights_keys(orc)
    for c in (False, True):
        yield lambda c=c: mask_pins.test_statistics(orc, c)
    yield lambda: mask_pins.test_fully_hidden_rows(orc)
    yield lambda: mask_pins.test_broadcast_strides_equal_materialised(orc)


def _first_failure(orc):
    for check in _battery(orc):
        try:
            check()
        except AssertionError as e:
            return e
    return None


def test_unmutated_oracle_passes_the_battery():
    assert _first_failure(oracle.get()) is None


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found once"
    path = tmp_path / f"mut_{name}.c"
    path.write_text(src.replace(old, new))
    lib = oracle.build(force=True, src=str(path), out=str(tmp_path / f"lib{name}.so"))
    assert _first_failure(oracle.Oracle(lib)) is not None, \
        f"no pin failed with the planted mistake {name!r}"
