"""The oracle's pins must catch plausible mistakes.

Each case copies ``oracle.c`` to a temporary directory, plants one mistake by text
substitution, builds it, points the oracle wrapper at the mutant and runs the pin tests:
at least one of them must fail.  Nothing here touches a GPU.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "nibble order swapped": ("int n = high ? (byte >> 4) : (byte & 0xF);",
                             "int n = high ? (byte & 0xF) : (byte >> 4);"),
    "nibbles not sign-extended": ("return n >= 8 ? n - 16 : n;", "return n;"),
    "scale as multiply by 7/m": ("float s = m / 7.0f;", "float s = m * (1.0f / 7.0f);"),
    "round half away from zero": ("v = rintf(row[c] / s);", "v = roundf(row[c] / s);"),
    "gate and up exchanged": ("h[r] = g / (1.0 + exp(-g)) * u;", "h[r] = u / (1.0 + exp(-u)) * g;"),
    "silu dropped": ("h[r] = g / (1.0 + exp(-g)) * u;", "h[r] = g * u;"),
    "down matrix transposed": ("acc += weight_at(wk, ex->down, ex->down_scale, j, r, f) * h[r];",
                               "acc += weight_at(wk, ex->down, ex->down_scale, r % d, j % f, f) * h[r];"),
    "bias enters the weights": ("for (int r = 0; r < k; ++r) sum += 1.0 / (1.0 + exp(-logit[idx[r]]));",
                                "for (int r = 0; r < k; ++r) sum += 1.0 / (1.0 + exp(-logit[idx[r]])) + "
                                "(L->router_bias ? L->router_bias[idx[r]] : 0.0);"),
    "ties go to the higher index": ("if (!taken[e] && (best < 0 || key[e] > key[best])) best = e;",
                                    "if (!taken[e] && (best < 0 || key[e] >= key[best])) best = e;"),
    "routed scaling dropped": ("w[r] = L->scaling * (1.0 / (1.0 + exp(-logit[idx[r]]))) / sum;",
                               "w[r] = (1.0 / (1.0 + exp(-logit[idx[r]]))) / sum;"),
    "shared expert dropped": ("for (int j = 0; j < d; ++j) o[j] += y[j];", "(void)0;"),
    "softmax over all experts": ("for (int r = 0; r < k; ++r) sum += exp(logit[idx[r]] - m);",
                                 "for (int e = 0; e < E; ++e) sum += exp(logit[e] - m);"),
    "int2 codes read highest bits first": ("int n = (byte >> (2 * i)) & 3;", "int n = (byte >> (6 - 2 * i)) & 3;"),
    "int2 codes not sign-extended": ("return n >= 2 ? n - 4 : n;", "return n;"),
    "int2 packer reverses the byte": ("b |= (uint8_t)((q[r * cols + 4 * j + i] & 3) << (2 * i));",
                                      "b |= (uint8_t)((q[r * cols + 4 * j + i] & 3) << (6 - 2 * i));"),
    "tier qmax off by one": ("const float qmax = (float)((1 << (bits - 1)) - 1);",
                             "const float qmax = (float)(1 << (bits - 1));"),
    "group score is the best key only": ("score[g] = per >= 2 ? b1 + b2 : b1;", "score[g] = b1;"),
    "equal group scores go to the higher group": (
        "if (!keep[g] && (best < 0 || score[g] > score[best])) best = g;",
        "if (!keep[g] && (best < 0 || score[g] >= score[best])) best = g;"),
    "top-p needs a share above p": ("if (cum / total >= p) { m = r + 1; break; }",
                                    "if (cum / total > p) { m = r + 1; break; }"),
    "top-p keeps the weights unscaled": ("w[r] = w[r] * (total / kept);", "w[r] = w[r];"),
}

PIN_TESTS = [
    lambda: pins.test_nibble_layout_golden(),
    lambda: pins.test_quantiser_golden_rows(),
    lambda: pins.test_topk_brute_force_tiny("tiny", 64),
    lambda: pins.test_topk_sigmoid_brute_force_with_bias(),
    lambda: pins.test_exact_ties_go_to_lower_index(),
    lambda: pins.test_gate_weights_closed_forms(),
    lambda: pins.test_bias_changes_selection_not_weights(),
    lambda: pins.test_single_expert_layer_is_textbook_swiglu(oracle.W_INT4),
    lambda: pins.test_single_expert_layer_is_textbook_swiglu(oracle.W_BF16),
    lambda: pins.test_shared_expert_adds_with_weight_one(),
    lambda: pins.test_exact_integer_case(),
    lambda: pins.test_int4_packing_bit_identical_to_int8_container((33, 130)),
    lambda: pins.test_int2_crumb_layout_golden(),
    lambda: pins.test_tier_quantiser_golden_rows("int2_rows"),
    lambda: pins.test_tier_quantiser_golden_rows("int8_rows"),
    lambda: pins.test_int2_packing_bit_identical_to_int8_container((33, 132)),
    lambda: pins.test_single_expert_layer_is_textbook_swiglu_other_tiers(oracle.W_INT2, 2),
    lambda: pins.test_grouped_selection_golden(),
    lambda: pins.test_grouped_selection_brute_force(oracle.ROUTER_SIGMOID),
    lambda: pins.test_top_p_golden(),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    mutated = src.replace(old, new)
    c = tmp_path / "oracle_mutant.c"
    so = tmp_path / "liboracle_mutant.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-std=c11", "-fPIC", "-shared",
                           str(c), "-o", str(so), "-lm"])
    real = oracle.lib()
    mutant = ctypes.CDLL(str(so))
    for fn in ("oracle_quantize_int8", "oracle_pack_int4", "oracle_unpack_int4", "oracle_route",
               "oracle_forward", "oracle_expert_ffn", "oracle_num_threads", "oracle_quantize_tier",
               "oracle_pack_int2", "oracle_unpack_int2"):
        getattr(mutant, fn).argtypes = getattr(real, fn).argtypes
        getattr(mutant, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", mutant)
    failed = 0
    for pin in PIN_TESTS:
        try:
            pin()
        except (AssertionError, RuntimeError):
            failed += 1
    assert failed >= 1, f"no pin caught the mutant '{name}'"
