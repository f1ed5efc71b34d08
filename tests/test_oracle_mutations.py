"""Plant plausible mistakes in the oracle and check that its pins catch them.

Each case copies oracle/moe_oracle.c, applies one textual change (a flipped
tie-break, an off-by-one in the capacity, a dropped factor, ...), builds the
copy into a temporary library, points the oracle module at it and runs the
pin tests that should notice. A mutation that no pin notices fails this test:
it would be a mistake the oracle could carry unnoticed.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_backward as bwd_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

# (name, original text, mutated text, pin tests expected to fail)
MUTATIONS = [
    ("tie-break favours the higher index",
     "return (a->idx < b->idx) ? -1 : (a->idx > b->idx);",
     "return (a->idx > b->idx) ? -1 : (a->idx < b->idx);",
     ["test_all_equal_keys_pick_lowest_indices", "test_tc_topk_matches_brute_force"]),
    ("capacity admits one assignment too many",
     "if (cap < 0 || used[e] < cap) {",
     "if (cap < 0 || used[e] <= cap) {",
     ["test_capacity_closed_forms", "test_capacity_all_equal_scores_worked_shape"]),
    ("group score keeps only the best key",
     "for (int j = 0; j < group_topn; ++j) sum = sum + tmp[j].key;",
     "for (int j = 0; j < 1; ++j) sum = sum + tmp[j].key;",
     ["test_group_limited_by_construction"]),
    ("normalised weights use the biased keys",
     "for (int j = 0; j < K; ++j) denom += (double)s[cand[j].idx];",
     "for (int j = 0; j < K; ++j) denom += (double)cand[j].key;",
     ["test_selection_only_bias"]),
    ("balance loss drops the factor E",
     "*lb = lb_coef * E * sum;",
     "*lb = lb_coef * sum;",
     ["test_lb_loss_is_coefficient_at_perfect_balance"]),
    ("z-loss of lse, not lse squared",
     "for (int t = 0; t < n; ++t) zz += lse[t] * lse[t];",
     "for (int t = 0; t < n; ++t) zz += lse[t];",
     ["test_z_loss_of_zero_logits"]),
    ("GELU with u / 2 instead of u / sqrt(2)",
     "return 0.5 * u * (1.0 + erf(u / sqrt(2.0)));",
     "return 0.5 * u * (1.0 + erf(u / 2.0));",
     ["test_expert_ffn_against_torch"]),
    ("combine ignores the gate",
     "double g = pair_gate[p];",
     "double g = 1.0;",
     ["test_ec_layer_matches_onehot_formulation"]),
    ("bias update with the sign flipped",
     "if (diff > 0)\n      bias[e] = bias[e] - rate;",
     "if (diff > 0)\n      bias[e] = bias[e] + rate;",
     ["test_bias_update_two_expert_example"]),
    ("bf16 rounding via fp32 (double rounding)",
     "double q = ldexp(v, -ulp_exp);",
     "double q = ldexp((double)(float)v, -ulp_exp);",
     ["test_round_bf16_against_torch_and_ties"]),
    ("router adds the logit bias twice",
     "if (logit_bias) v += (double)logit_bias[e];",
     "if (logit_bias) v += 2.0 * (double)logit_bias[e];",
     ["test_router_against_library"]),
    ("sqrt(softplus) score without the square root",
     "        s = sqrt(sp);",
     "        s = sp;",
     ["test_sqrtsoftplus_closed_forms"]),
    ("SwiGLU up value from W1 instead of W3",
     "        for (int i = 0; i < d; ++i) b += (double)x[i] * (double)W3[(size_t)j * d + i];",
     "        for (int i = 0; i < d; ++i) b += (double)x[i] * (double)W1[(size_t)j * d + i];",
     ["test_expert_ffn_against_torch"]),
    ("down projection reads W2 transposed",
     "      for (int j = 0; j < h; ++j) y += (double)W2[(size_t)i * h + j] * (double)H[j];",
     "      for (int j = 0; j < h; ++j) y += (double)W2[(size_t)j * d + i] * (double)H[j];",
     ["test_expert_ffn_against_torch"]),
    ("router reads W_g transposed",
     "      for (int e = 0; e < E; ++e) acc[e] += x * (double)w[e];",
     "      for (int e = 0; e < E; ++e) acc[e] += x * (double)Wg[(size_t)e * d + i] + 0.0 * w[e];",
     ["test_router_against_library"]),
    ("top-k keeps the smallest keys",
     "  if (a->key > b->key) return -1;\n  if (a->key < b->key) return 1;",
     "  if (a->key < b->key) return -1;\n  if (a->key > b->key) return 1;",
     ["test_tc_topk_matches_brute_force", "test_ec_topk_matches_brute_force"]),
    # backward pass
    ("SwiGLU backward drops the u (1 - sigma) part of silu'",
     "dUs[j] = round_store(dh * vs * sg * (1.0 + us * (1.0 - sg)), store);",
     "dUs[j] = round_store(dh * vs * sg, store);",
     ["test_backward_matches_finite_differences", "test_expert_backward_against_autograd"]),
    ("expert input gradient misses the W3 path",
     "        for (int j = 0; j < h; ++j) a += (double)dVs[j] * (double)W3[(size_t)j * d + i];",
     "        for (int j = 0; j < h; ++j) a += 0.0 * (double)dVs[j];",
     ["test_backward_matches_finite_differences", "test_expert_backward_against_autograd"]),
    ("GELU backward without the u phi(u) term",
     "return 0.5 * (1.0 + erf(u / sqrt(2.0))) + u * exp(-0.5 * u * u) / sqrt(2.0 * pi);",
     "return 0.5 * (1.0 + erf(u / sqrt(2.0))) + 0.0 * pi;",
     ["test_backward_matches_finite_differences", "test_expert_backward_against_autograd"]),
    ("combine backward forgets the gate in dY",
     "dY[(size_t)p * d + i] = round_store(gate * go, store);",
     "dY[(size_t)p * d + i] = round_store(go + 0.0 * gate, store);",
     ["test_backward_matches_finite_differences"]),
    ("softmax backward without the <S, dS> term",
     "for (int e = 0; e < E; ++e) out[e] = (double)s[e] * (g[e] - dot);",
     "for (int e = 0; e < E; ++e) out[e] = (double)s[e] * g[e] + 0.0 * dot;",
     ["test_backward_matches_finite_differences",
      "test_score_and_router_backward_against_autograd"]),
    ("sigmoid backward as s instead of s (1 - s)",
     "for (int e = 0; e < E; ++e) out[e] = g[e] * (double)s[e] * (1.0 - (double)s[e]);",
     "for (int e = 0; e < E; ++e) out[e] = g[e] * (double)s[e];",
     ["test_backward_matches_finite_differences",
      "test_score_and_router_backward_against_autograd"]),
    ("sqrt(softplus) backward without the 1/2",
     "out[e] = g[e] * sigm((double)L[e]) / (2.0 * (double)s[e]);",
     "out[e] = g[e] * sigm((double)L[e]) / (double)s[e];",
     ["test_backward_matches_finite_differences",
      "test_score_and_router_backward_against_autograd"]),
    ("z-loss gradient without the factor 2",
     "out[e] += z_coef * 2.0 * lse[t] / n * exp((double)L[e] - lse[t]);",
     "out[e] += z_coef * lse[t] / n * exp((double)L[e] - lse[t]);",
     ["test_backward_matches_finite_differences",
      "test_score_and_router_backward_against_autograd"]),
    ("balance-loss gradient not divided by n",
     "g[e] += lb_coef * E * ((double)load[e] / ((double)n * K)) / n;",
     "g[e] += lb_coef * E * ((double)load[e] / ((double)n * K));",
     ["test_backward_matches_finite_differences",
      "test_score_and_router_backward_against_autograd"]),
    ("normalised weights backward without the sum w dw term",
     "for (int j = 0; j < K; ++j) ds[it[j]] += (g[j] - dot) / sum;",
     "for (int j = 0; j < K; ++j) ds[it[j]] += (g[j] + 0.0 * dot) / sum;",
     ["test_backward_matches_finite_differences", "test_normalized_gate_backward_closed_form"]),
    ("expert choice gate read from the wrong expert",
     "G[(size_t)e * k + j] = S[(size_t)col[j].idx * E + e];",
     "G[(size_t)e * k + j] = S[(size_t)col[j].idx * E + (e + 1) % E];",
     ["test_ec_every_expert_holds_exactly_k_distinct"]),
]


def _build_mutant(tmp_path, original, mutated):
    src = open(SRC).read()
    assert src.count(original) == 1, f"mutation anchor not unique: {original!r}"
    path = tmp_path / "moe_oracle.c"
    path.write_text(src.replace(original, mutated))
    (tmp_path / "moe_oracle.h").write_text(
        open(os.path.join(os.path.dirname(SRC), "moe_oracle.h")).read())
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-o", str(lib), str(path), "-lm"])
    return str(lib)


def _run_pin(name):
    """Run every parametrisation of a pin test; True if all of them pass."""
    fn = getattr(pins, name, None) or getattr(bwd_pins, name)
    params = getattr(fn, "pytestmark", [])
    cases = [{}]
    for m in params:
        if m.name == "parametrize":
            argnames, values = m.args[0], m.args[1]
            argnames = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) \
                else list(argnames)
            new = []
            for c in cases:
                for v in values:
                    v = v if len(argnames) > 1 else (v,)
                    new.append({**c, **dict(zip(argnames, v))})
            cases = new
    for kw in cases:
        try:
            fn(**kw)
        except AssertionError:
            return False
    return True


@pytest.mark.parametrize("name,original,mutated,catchers", MUTATIONS,
                         ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, name, original, mutated, catchers):
    lib = _build_mutant(tmp_path, original, mutated)
    oracle.use_library(lib)
    try:
        caught = [c for c in catchers if not _run_pin(c)]
    finally:
        oracle.use_library(None)
    assert caught, f"no pin caught the planted mistake: {name}"


def test_unmutated_oracle_passes_the_same_pins():
    for _, _, _, catchers in MUTATIONS:
        for c in catchers:
            assert _run_pin(c), c
