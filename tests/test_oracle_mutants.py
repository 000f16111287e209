"""The oracle's pins catch plausible mistakes.

Each mutant below is a copy of oracle/moe_oracle.c with one plausible error
planted in it (a flipped sign, a transposed operand, a dropped term, a wrong
tie-break or order).  It is compiled into a temporary library on the CPU and
run against the pin tests of test_oracle_pins.py; every mutant must make at
least one pin fail.  No GPU is used.
"""
import importlib.util
import os
import subprocess
import sys
import tempfile

import pytest

import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "silu_sign": ("hbuf[i] = g / (1.0 + exp(-g)) * u;", "hbuf[i] = g / (1.0 + exp(g)) * u;"),
    "gate_up_swapped": ("hbuf[i] = g / (1.0 + exp(-g)) * u;", "hbuf[i] = u / (1.0 + exp(-u)) * g;"),
    "down_transposed": ("for (int32_t i = 0; i < I; ++i) a += bf16_to_f64(rd[i]) * hbuf[i];",
                        "for (int32_t i = 0; i < I; ++i) a += bf16_to_f64(wd[((size_t)i * H + o) % ((size_t)H * I)]) * hbuf[i];"),
    "shared_term_dropped": ("for (int32_t c = 0; c < H; ++c) o[c] += s * y[c];",
                            "for (int32_t c = 0; c < H; ++c) o[c] += 0.0 * s * y[c];"),
    "shared_gate_sign": ("return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));"),
    "topk_tie_higher_id": ("if (best < 0 || l[e] > l[best]) best = e;", "if (best < 0 || l[e] >= l[best]) best = e;"),
    "topk_ascending": ("if (best < 0 || l[e] > l[best]) best = e;", "if (best < 0 || l[e] < l[best]) best = e;"),
    "no_renormalisation": ("if (norm_topk)\n            for (int32_t j = 0; j < k; ++j) w[(size_t)t * k + j] = w[(size_t)t * k + j] / ws;",
                           "if (norm_topk && 0)\n            for (int32_t j = 0; j < k; ++j) w[(size_t)t * k + j] = w[(size_t)t * k + j] / ws;"),
    "softmax_no_normalise": ("for (int32_t e = 0; e < E; ++e) p[e] = p[e] / s;", "for (int32_t e = 0; e < E; ++e) p[e] = p[e];"),
    "budget_keeps_lightest": ("if (x->agg > y->agg) return -1;   /* descending aggregate weight */\n    if (x->agg < y->agg) return 1;",
                              "if (x->agg > y->agg) return 1;\n    if (x->agg < y->agg) return -1;"),
    "budget_counts_not_weights": ("agg[idx[(size_t)t * k + j]] += w[(size_t)t * k + j];",
                                  "agg[idx[(size_t)t * k + j]] += 1.0f;"),
    "budget_tie_higher_id": ("return (x->id < y->id) ? -1 : (x->id > y->id); /* equal -> lower id first */",
                             "return (x->id > y->id) ? -1 : (x->id < y->id);"),
    "budget_no_renorm": ("if (norm_topk && c > 0 && c < keff[t]) {", "if (norm_topk && c > 0 && c < 0) {"),
    "budget_renorm_all": ("if (norm_topk && c > 0 && c < keff[t]) {", "if (norm_topk && c > 0 && c <= k) {"),
    "budget_renorm_by_k": ("if (norm_topk && c > 0 && c < keff[t]) {", "if (norm_topk && c > 0 && c < k) {"),
    "router_transposed": ("a += bf16_to_f64(x[(size_t)t * H + h]) * bf16_to_f64(wr[(size_t)e * H + h]);",
                          "a += bf16_to_f64(x[(size_t)t * H + h]) * bf16_to_f64(wr[((size_t)h * E + e) % ((size_t)E * H)]);"),
    "router_skips_first": ("for (int32_t h = 0; h < H; ++h)\n                a += bf16_to_f64(x",
                           "for (int32_t h = 1; h < H; ++h)\n                a += bf16_to_f64(x"),
    "topp_strict": ("if (j > 0 && mass >= topp) { c = j; break; }", "if (j > 0 && mass > topp) { c = j; break; }"),
    "topp_drops_crossing_slot": ("                if (j > 0 && mass >= topp) { c = j; break; }\n                mass += tw[j];",
                                 "                mass += tw[j];\n                if (j > 0 && mass >= topp) { c = j; break; }"),
    "topp_no_renorm": ("if (norm_topk && c < k) {", "if (norm_topk && c < 0) {"),
    "forward_skips_topp": ("rc = oracle_topp(T, k, norm_topk, topp, idx, w, keff);",
                           "rc = oracle_topp(T, k, norm_topk, 0.0f, idx, w, keff);"),
    "budget_off_by_one": ("if (N == 0 || nu <= N) return ORACLE_OK;", "if (N == 0 || nu <= N + 1) return ORACLE_OK;"),
    "dispatch_tokens_descending": ("        for (int32_t t = 0; t < T; ++t)\n            for (int32_t j = 0; j < keff[t]; ++j)\n                if (idx[(size_t)t * k + j] == e) {",
                                   "        for (int32_t t = T - 1; t >= 0; --t)\n            for (int32_t j = 0; j < keff[t]; ++j)\n                if (idx[(size_t)t * k + j] == e) {"),
    "combine_wrong_weight": ("double wj = (double)w[(size_t)t * k + j];", "double wj = (double)w[(size_t)t * k + (j + 1) % k];"),
    "ffn_params_two_matrices": ("int64_t oracle_ffn_params(int64_t H, int64_t I) { return 3 * H * I; }",
                                "int64_t oracle_ffn_params(int64_t H, int64_t I) { return 2 * H * I; }"),
}

# every pin test with the arguments it is run with
PINS = [
    ("test_param_counts_match_drafter_table", {}),
    ("test_router_logits_unit_vectors_and_torch", {}),
    ("test_route_closed_form_worked_example", {}),
    ("test_route_ties_take_lower_id", {}),
    ("test_route_brute_force_topk", dict(E=8, k=3)),
    ("test_route_weights_against_torch_softmax", {}),
    ("test_route_k_equals_E_is_full_softmax", {}),
    ("test_budget_worked_example", {}),
    ("test_budget_brute_force_keeps_heaviest_subset", dict(seed=0)),
    ("test_budget_invariants", dict(norm=True)),
    ("test_budget_drops_can_empty_tokens", {}),
    ("test_topp_worked_example", {}),
    ("test_topp_invariants", dict(norm=True)),
    ("test_topp_then_budget_composition", {}),
    ("test_forward_routes_topp_then_budget", dict(N=4, p=0.8)),
    ("test_dispatch_matches_stable_sort", dict(T=33, E=16, k=4, N=5)),
    ("test_ffn_closed_form_unit_vectors", {}),
    ("test_ffn_single_expert_is_plain_swiglu_mlp", {}),
    ("test_combine_k_equals_E_is_softmax_mixture", {}),
    ("test_forward_dense_masked_loop", dict(N=3, norm=True)),
    ("test_shared_gate_closed_form", {}),
]


def _load_mutant(name, tmp):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutant {name}: anchor not found exactly once"
    path_c = os.path.join(tmp, f"{name}.c")
    path_so = os.path.join(tmp, f"lib{name}.so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    quant_c = os.path.join(ROOT, "oracle", "quant_oracle.c")  # the rest of the oracle library, unchanged
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", path_c, quant_c, "-o", path_so, "-lm"],
                   check=True)
    # a fresh copy of the oracle wrapper module bound to the mutant library
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{name}", os.path.join(ROOT, "oracle", "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod  # dataclasses resolve their module by name
    spec.loader.exec_module(mod)
    mod._LIB = path_so
    mod.build = lambda force=False: path_so
    return mod


@pytest.fixture(scope="module")
def tmpdir_mod():
    with tempfile.TemporaryDirectory() as d:
        yield d


def test_unmutated_oracle_passes_every_pin(oracle_mod):
    for fn, kw in PINS:
        getattr(pins, fn)(oracle_mod, **kw)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmpdir_mod):
    mod = _load_mutant(name, tmpdir_mod)
    failed = []
    for fn, kw in PINS:
        try:
            getattr(pins, fn)(mod, **kw)
        except AssertionError:
            failed.append(fn)
    assert failed, f"no pin caught the mutant {name}"
    print(name, "caught by", failed)
