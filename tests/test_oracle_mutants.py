"""Plant plausible mistakes in a copy of the oracle's C source (on the CPU)
and check that the pin suite catches every one.  This is what makes the pins
worth trusting: a dropped term, a wrong index, a wrong sign, swapped operand
roles or a broken decoder each fail at least one pin."""
import os

import pytest

import oracle
import oracle_pins

# (name, original text, planted mistake).  Each original must occur exactly
# once in the committed source, so a change there breaks this test loudly.
MUTANTS = [
    ("dropped_first_term",
     "for (int64_t k = 0; k < K; ++k) {\n        double pg",
     "for (int64_t k = 1; k < K; ++k) {\n        double pg"),
    ("reversed_weight_index",
     "double pg = x[k] * wg[k];", "double pg = x[k] * wg[K - 1 - k];"),
    ("gate_up_swapped",
     "if (h_out) *h_out = oracle_act(alpha * g, act) * u;",
     "if (h_out) *h_out = oracle_act(alpha * u, act) * g;"),
    ("multiplier_after_activation",
     "if (h_out) *h_out = oracle_act(alpha * g, act) * u;",
     "if (h_out) *h_out = alpha * oracle_act(g, act) * u;"),
    ("gelu_sign",
     "return x * oracle_sigmoid(2.0 * y);", "return x * oracle_sigmoid(-2.0 * y);"),
    ("dgelu_complement",
     "double oms = oracle_sigmoid(-2.0 * y);", "double oms = oracle_sigmoid(2.0 * y);"),
    ("gelu_slope_cubic_term",
     "double dy = ORACLE_GELU_C * (1.0 + 3.0 * ORACLE_GELU_A * x * x);",
     "double dy = ORACLE_GELU_C * (1.0 + ORACLE_GELU_A * x * x);"),
    ("dG_missing_multiplier",
     "*dg = dh * u * alpha * oracle_dact(alpha * g, act);",
     "*dg = dh * u * oracle_dact(alpha * g, act);"),
    ("sigmoid_sign",
     "return 1.0 / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(x));"),
    ("dsilu_sign",
     "return s * (1.0 + x * (1.0 - s));", "return s * (1.0 - x * (1.0 - s));"),
    ("dU_uses_up_operand",
     "*du = dh * oracle_act(alpha * g, act);", "*du = dh * oracle_act(alpha * u, act);"),
    ("wrong_weight_row",
     "one_output(X + m * K, Wg + n * K, Wu + n * K, K,",
     "one_output(X + m * K, Wg + ((n + 1) % N) * K, Wu + n * K, K,"),
    ("dx_wrong_weight",
     "acc += dG[m * N + n] * Wg[n * K + k] + dU[m * N + n] * Wu[n * K + k];",
     "acc += dG[m * N + n] * Wu[n * K + k] + dU[m * N + n] * Wg[n * K + k];"),
    ("dw_transposed_index",
     "ag += dG[m * N + n] * X[m * K + k];", "ag += dG[m * N + n] * X[m * K + (K - 1 - k)];"),
    ("e4m3_ties_to_odd",
     "(d == best_d && (c & 1) == 0 && (best & 1) == 1)", "(d == best_d && (c & 1) == 1 && (best & 1) == 0)"),
    ("ue8m0_off_by_one",
     "while (e < 127 && amax > 448.0 * ldexp(1.0, e))", "while (e < 127 && amax >= 448.0 * ldexp(1.0, e))"),
    ("quant_block_16",
     "int64_t lo = b * 32, hi = lo + 32 < n ? lo + 32 : n;", "int64_t lo = b * 32, hi = lo + 16 < n ? lo + 16 : n;"),
    ("e4m3_exponent_bias",
     "v = ldexp(1.0 + (double)mf / 8.0, ef - 7);", "v = ldexp(1.0 + (double)mf / 8.0, ef - 8);"),
    ("bf16_decode_shift",
     "uint32_t u = ((uint32_t)b) << 16;", "uint32_t u = ((uint32_t)b) << 15;"),
    ("magnitude_missing_abs",
     "ag += fabs(pg);", "ag += pg;"),
]


@pytest.mark.parametrize("name,orig,bad", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, orig, bad):
    src = open(oracle.SOURCE).read()
    assert src.count(orig) == 1, f"mutation anchor for {name} not unique/found"
    mutated = tmp_path / f"oracle_{name}.c"
    mutated.write_text(src.replace(orig, bad))
    lib = oracle.compile_source(str(mutated), str(tmp_path / f"lib_{name}.so"))
    m = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(m)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
