"""Planted-mistake checks for the oracle's pins (CPU only).

Each case copies attention_ref.c, plants one plausible mistake (a transposed
operand, a wrong head map, a dropped scale, an off-by-one mask, a wrong log
base, a wrong exponent bias, the wrong rounding rule), builds the copy with
gcc and runs the pins against it: at least one pin must fail.  The planted
copies live in a temporary directory; the committed oracle is untouched."""
import os

import pytest

import oracle
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
    "scale_dropped": ("s[j] = scale * acc;", "s[j] = acc;"),
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
    "online_stale_max": ("d = d * exp(m - m_new) + exp(x[i] - m_new);",
                         "d = d + exp(x[i] - m_new);"),
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
