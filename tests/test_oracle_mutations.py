"""The pins must catch plausible mistakes in the oracle.

Each case below compiles a copy of the oracle's C source with one deliberate
mistake (a dropped term, a wrong sign, a transposed operand, a wrong index or
tie rule) into a temporary directory, points the oracle wrapper at it, and
requires that at least one pin of tests/test_oracle_pins.py fails.  Everything
runs on the CPU; the real oracle is restored afterwards.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "lmoe_oracle.c")

PIN_FUNCS = [
    pins.test_golden_hand_case_b,
    pins.test_golden_hand_case_relu2,
    pins.test_alpha_one_relu2_is_the_pages_moe_class,
    pins.test_golden_silu_sign_and_gate_role,
    lambda: pins.test_topk_brute_force(7, 3),
    pins.test_topk_ties_go_to_lower_index,
    pins.test_gates_sum_to_one_and_are_non_increasing,
    pins.test_router_bias_enters_before_softmax,
    lambda: pins.test_dense_limit_K_equals_N("swiglu"),
    pins.test_alpha_one_identity_projections_is_standard_moe,
    lambda: pins.test_mask_form_over_all_experts("swiglu"),
    lambda: pins.test_dispatch_is_the_unique_stable_grouping(37, 4, 16),
]

MUTATIONS = {
    "silu_sign": ("return a / (1.0 + exp(-a));", "return a / (1.0 + exp(a));"),
    "gate_up_swapped": ("a[j] = silu(a[j]) * b[j];", "a[j] = silu(b[j]) * a[j];"),
    "no_renormalise": ("for (int k = 0; k < K; ++k) gates[k] /= psum;",
                       "for (int k = 0; k < K; ++k) gates[k] /= 1.0;"),
    "ties_to_higher_index": ("if (best < 0 || s[e] > s[best]) best = e;",
                             "if (best < 0 || s[e] >= s[best]) best = e;"),
    "smallest_selected": ("if (best < 0 || s[e] > s[best]) best = e;",
                          "if (best < 0 || s[e] < s[best]) best = e;"),
    "all_matrices_transposed": ("size_t base = off + (size_t)r * (size_t)cols;\n"
                                "    for (int c = 0; c < cols; ++c) acc += elem(W, dt, base + (size_t)c) * v[c];",
                                "for (int c = 0; c < cols; ++c) acc += elem(W, dt, off + (size_t)c * rows + r) * v[c];"),
    "shared_dropped": ("for (int i = 0; i < d; ++i) yr[i] += sh[i];",
                       "for (int i = 0; i < d; ++i) yr[i] += 0.0 * sh[i];"),
    "slot_gate_index": ("for (int i = 0; i < l; ++i) u[i] += g[k] * eo[i];",
                        "for (int i = 0; i < l; ++i) u[i] += g[0] * eo[i];"),
    "relu2_without_square": ("static double relu2(double a) { return a > 0.0 ? a * a : 0.0; }",
                             "static double relu2(double a) { return a > 0.0 ? a : 0.0; }"),
    "relu2_without_relu": ("static double relu2(double a) { return a > 0.0 ? a * a : 0.0; }",
                           "static double relu2(double a) { return a * a; }"),
    "bias_dropped": ("s[e] = acc + (L->b_router ? L->b_router[e] : 0.0);", "s[e] = acc;"),
    "dispatch_token_descending": ("for (int64_t t = 0; t < T; ++t)\n      for (int k = 0; k < K; ++k)\n        if (ids[t * K + k] == e) {",
                                  "for (int64_t t = T - 1; t >= 0; --t)\n      for (int k = 0; k < K; ++k)\n        if (ids[t * K + k] == e) {"),
    "softmax_over_selected_only_wrong_denominator": ("gates[k] = exp(s[ids[k]] - smax) / denom; /* p_{id_k} */\n    psum += gates[k];",
                                                     "gates[k] = exp(s[ids[k]]) / denom; /* p_{id_k} */\n    psum += 1.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new, 1))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(lib), str(mutated), "-lm"])
    oracle._swap_library(str(lib))
    try:
        caught = []
        for f in PIN_FUNCS:
            try:
                f()
            except (AssertionError, ValueError):
                caught.append(getattr(f, "__name__", "lambda"))
        assert caught, f"no pin caught mutation {name}"
    finally:
        oracle._swap_library(None)
