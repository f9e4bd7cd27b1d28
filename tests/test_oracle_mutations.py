"""The pins must catch plausible mistakes in the oracle.

Each case copies the C++ oracle's source, plants one mistake in the copy (a
dropped term, a wrong sign, index or bit field, a transposed operand), compiles
it into a temporary library on the CPU, points the `oracle` functions at that
build for the duration of the case, and checks that at least one pin fails.
The committed oracle is never modified.
"""
import concurrent.futures
import os

import pytest

import oracle
import oracle.cpp as ocpp
from oracle import build as obuild
from tests import test_oracle_pins as pins

# (name, exact text in pi_oracle.cpp, replacement); each text occurs once
MUTANTS = [
    ("predict-no-relu", "a[(size_t)b * r + j] = z[b] > 0.0 ? z[b] : 0.0;",
     "a[(size_t)b * r + j] = z[b];"),
    ("predict-no-b2", "z[b] += L->b2[n];", "(void)0;"),
    ("predict-no-b1", "if (L->b1) z[b] += L->b1[j];", "(void)0;"),
    ("predict-tie-active", "z[b] > L->threshold ? 1 : 0", "z[b] >= L->threshold ? 1 : 0"),
    ("predict-x-transposed", "xt[(size_t)k * B + b] = x[(size_t)b * d + k];",
     "xt[(size_t)k * B + b] = x[(size_t)k * B + b];"),
    ("masked-row-by-position", "widen_row(L->w_down_t, L->wdtype, idx[k], d, row.data());",
     "widen_row(L->w_down_t, L->wdtype, k, d, row.data());"),
    ("masked-h-transposed", "const double hb = h[(size_t)b * K + k];",
     "const double hb = h[(size_t)k * B + b];"),
    ("reglu-gate-up-swapped",
     "widen_row(L->w_up, L->wdtype, i, d, up.data());\n    if (L->act == 1) widen_row(L->w_gate, L->wdtype, i, d, gate.data());",
     "widen_row(L->act == 1 ? L->w_gate : L->w_up, L->wdtype, i, d, up.data());\n    if (L->act == 1) widen_row(L->w_up, L->wdtype, i, d, gate.data());"),
    ("relu-drop-bias", "if (L->b_up) ub += L->b_up[i];", "(void)0;"),
    ("reglu-drop-bias", "if (L->b_gate) gb += L->b_gate[i];", "(void)0;"),
    ("reglu-no-relu", "v = (gb > 0.0 ? gb : 0.0) * u[b];", "v = gb * u[b];"),
    ("sqrelu-unsquared", "v = L->act == 2 ? rl * rl : rl;", "v = rl;"),
    ("q4-nibbles-swapped", "const int lo = p[2 + j] & 0x0f;\n      const int hi = p[2 + j] >> 4;",
     "const int hi = p[2 + j] & 0x0f;\n      const int lo = p[2 + j] >> 4;"),
    ("q4-offset-7", "out[blk * 32 + j] = (double)(lo - 8) * scale;",
     "out[blk * 32 + j] = (double)(lo - 7) * scale;"),
    ("q4-scale-big-endian", "(uint16_t)(p[0] | (p[1] << 8))", "(uint16_t)((p[0] << 8) | p[1])"),
    ("union-is-intersection",
     "bool any = false;\n    for (int b = 0; b < B; ++b) any = any || mask[(size_t)b * F + n] != 0;",
     "bool any = true;\n    for (int b = 0; b < B; ++b) any = any && mask[(size_t)b * F + n] != 0;"),
    ("rms-no-eps", "std::sqrt(ss / d + 1e-6)", "std::sqrt(ss / d)"),
    ("rms-divisor", "std::sqrt(ss / d + 1e-6)", "std::sqrt(ss / (d - 1) + 1e-6)"),
    ("round-truncates", "std::nearbyint(std::ldexp(ax, -qe))", "std::trunc(std::ldexp(ax, -qe))"),
    ("round-ties-away", "std::nearbyint(std::ldexp(ax, -qe))", "std::round(std::ldexp(ax, -qe))"),
    ("bf16-exponent-shift-8", "std::ldexp((double)(128 + m), e - 134)",
     "std::ldexp((double)(128 + m), e - 126)"),
    ("bf16-read-as-f16", "const double* v = pattern_values(dtype).data();",
     "const double* v = pattern_values(0).data();"),
    ("bf16-fraction-7-as-8", "const int m = b & 0x7f;\n  double v;\n  if (e == 0) {\n    v = std::ldexp((double)m, -133);",
     "const int m = b & 0xff;\n  double v;\n  if (e == 0) {\n    v = std::ldexp((double)m, -133);"),
    ("f16-subnormal-scale", "v = std::ldexp((double)m, -24);", "v = std::ldexp((double)m, -25);"),
    ("f16-bias-off-by-one", "std::ldexp((double)(1024 + m), e - 25)",
     "std::ldexp((double)(1024 + m), e - 24)"),
]

PIN_CASES = [
    (pins.test_predict_and_ffn_brute_force, dict(act="relu", shape=(16, 8, 4), wdtype="f16")),
    (pins.test_predict_and_ffn_brute_force, dict(act="reglu", shape=(48, 16, 6), wdtype="bf16")),
    (pins.test_predict_and_ffn_brute_force, dict(act="sqrelu", shape=(16, 8, 4), wdtype="f16")),
    (pins.test_predict_and_ffn_brute_force, dict(act="relu", shape=(64, 12, 8), wdtype="q4_0")),
    (pins.test_every_subset_closed_form, dict(act="relu", wdtype="f16")),
    (pins.test_every_subset_closed_form, dict(act="reglu", wdtype="bf16")),
    (pins.test_tie_is_inactive, {}),
    (pins.test_fig8_worked_example, {}),
    (pins.test_union_index_brute_force, {}),
    (pins.test_predictor_closed_form_pm_construction, {}),
    (pins.test_measured_sparsity_matches_profile, {}),
    (pins.test_q4_0_golden_block, {}),
    (pins.test_round_f16_ties_and_library, {}),
    (pins.test_round_bf16_ties_and_library, {}),
    (pins.test_round_overflow_and_subnormal_ties, {}),
    (pins.test_rms_cast_special_cases, {}),
    (pins.test_stack_brute_force, {}),
    (pins.test_widen_bf16_hand_patterns, {}),
    (pins.test_widen_f16_hand_patterns, {}),
]


def _mutated_source(old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor must occur once: {old!r}"
    return src.replace(old, new)


@pytest.fixture(scope="module")
def mutant_libs(tmp_path_factory):
    d = tmp_path_factory.mktemp("oracle_mutants")

    def make(m):
        name, old, new = m
        src = os.path.join(d, f"{name}.cpp")
        with open(src, "w") as f:
            f.write(_mutated_source(old, new))
        return name, obuild.compile_source(src, os.path.join(d, f"lib_{name}.so"))

    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        return dict(ex.map(make, MUTANTS))


def test_unmutated_oracle_passes_every_pin_case():
    for case, kw in PIN_CASES:
        case(**kw)


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(monkeypatch, mutant_libs, name):
    mut = ocpp.CppOracle(mutant_libs[name])
    for fn in ocpp.API:
        monkeypatch.setattr(oracle, fn, getattr(mut, fn))
    caught = None
    for case, kw in PIN_CASES:
        try:
            case(**kw)
        except (AssertionError, ValueError, FloatingPointError):
            caught = case.__name__
            break
    assert caught, f"no pin caught the planted mistake {name}"
