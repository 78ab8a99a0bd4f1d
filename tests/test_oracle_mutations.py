"""The oracle's pins catch plausible mistakes (no GPU).

Each case plants one plausible slip in a copy of the oracle's C source (a wrong
reading of a page's definition, a dropped term, a swapped index), compiles the
copy, points the oracle binding at it and runs the pins that should notice: at
least one of them must fail.  The product library is not involved; the planted
mistakes live only in a temporary copy of the oracle.
"""
import ctypes as C
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

# (name, original source text (must occur once), planted text, [(pin, kwargs), ...])
MUTATIONS = [
    ("softmax selection key on the biased logit (l' + B)",
     "key[e] = s[e] + (p->selection_bias ? (double)p->selection_bias[e] : 0.0);",
     "key[e] = (p->score == ORC_SOFTMAX ? (double)lp[e] : s[e]) + "
     "(p->selection_bias ? (double)p->selection_bias[e] : 0.0);",
     [("test_softmax_selection_bias_worked_example", {}),
      ("test_biased_selection_matches_brute_force_on_independent_keys",
       dict(score="softmax", E=12, k=4, renorm=True, S=2.5))]),
    ("softmax selection key as softmax(l' + B)",
     "key[e] = s[e] + (p->selection_bias ? (double)p->selection_bias[e] : 0.0);",
     "key[e] = (p->score == ORC_SOFTMAX && p->selection_bias) ? "
     "exp((double)lp[e] + (double)p->selection_bias[e]) : "
     "s[e] + (p->selection_bias ? (double)p->selection_bias[e] : 0.0);",
     [("test_softmax_selection_bias_worked_example", {}),
      ("test_biased_selection_matches_brute_force_on_independent_keys",
       dict(score="softmax", E=9, k=3, renorm=False, S=1.0))]),
    ("selection bias ignored",
     "key[e] = s[e] + (p->selection_bias ? (double)p->selection_bias[e] : 0.0);",
     "key[e] = s[e];",
     [("test_softmax_selection_bias_worked_example", {}),
      ("test_selection_bias_changes_choice_not_weight", {})]),
    ("weights taken from the biased key",
     "w[j] = s[idx[j]];",
     "w[j] = key[idx[j]];",
     [("test_selection_bias_changes_choice_not_weight", {}),
      ("test_softmax_selection_bias_worked_example", {})]),
    ("group scored by its best expert only",
     "gscore[g] = per >= 2 ? key[b1] + key[b2] : key[b1];",
     "gscore[g] = key[b1];",
     [("test_group_limited_selection_matches_exhaustive_search", dict(sel_std=0.0)),
      ("test_biased_group_selection_matches_exhaustive_search_on_independent_keys",
       dict(score="sigmoid"))]),
    ("ties to the higher index",
     "  if (ka != kb) return ka > kb;\n  return ia < ib;",
     "  if (ka != kb) return ka > kb;\n  return ia > ib;",
     [("test_topk_matches_brute_force_with_ties", dict(E=8, k=3))]),
    ("renormalizing sum not clamped",
     "double den = sum > 0x1p-14 ? sum : 0x1p-14;",
     "double den = sum;",
     [("test_renormalize_clamp_binds_only_for_small_sigmoid_sums", {})]),
    ("routed scale dropped",
     "for (int64_t j = 0; j < k; j++) w[j] = w[j] * p->routed_scale;",
     ";",
     [("test_renormalized_weights_sum_to_one_times_scale", {}), ("test_routed_scale_is_linear", {})]),
    ("router bias dropped",
     "if (p->router_bias) l = l + load_f32(p->router_bias, p->logit_dtype, e);",
     ";",
     [("test_softmax_and_sigmoid_scores_match_scipy", {})]),
    ("gate and up halves swapped",
     "int64_t rg = p->gu_layout == ORC_INTERLEAVED ? 2 * f : f;\n"
     "      int64_t ru = p->gu_layout == ORC_INTERLEAVED ? 2 * f + 1 : F + f;",
     "int64_t ru = p->gu_layout == ORC_INTERLEAVED ? 2 * f : f;\n"
     "      int64_t rg = p->gu_layout == ORC_INTERLEAVED ? 2 * f + 1 : F + f;",
     [("test_single_expert_equals_textbook_ffn",
       dict(act="silu", alpha=1.0, beta=0.0, limit=0.0)),
      ("test_expert_worked_example", {})]),
    ("beta added to the gate instead of the up value",
     "return a * (u + p->beta);",
     "return (a + p->beta) * u;",
     [("test_single_expert_equals_textbook_ffn",
       dict(act="gelu_erf", alpha=1.0, beta=0.5, limit=0.0))]),
    ("down bias dropped",
     "if (bd) acc += load(bd, p->act_dtype, ee * d + o);",
     ";",
     [("test_single_expert_equals_textbook_ffn",
       dict(act="relu", alpha=1.0, beta=0.0, limit=0.0))]),
    ("weigh-inputs also weighs the output",
     "double wout = p->weigh_inputs ? 1.0 : w[j];",
     "double wout = w[j];",
     [("test_weigh_inputs_is_quadratic_for_identity_activation", {})]),
    ("e2m1 nibbles swapped",
     "int code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);",
     "int code = (c % 2 == 0) ? (byte >> 4) : (byte & 0xF);",
     [("test_mxfp4_experts_equal_dequantized_experts", {})]),
    ("shared expert's sigmoid gate dropped",
     "gate = sigmoid(dot);",
     "gate = 1.0 + 0.0 * dot;",
     [("test_shared_expert_with_sigmoid_gate", {})]),
    ("plain FFN multiplies by beta as the gated form does",
     "  case ORC_SILU: return g * sigmoid(p->alpha * g);",
     "  case ORC_SILU: return g * sigmoid(p->alpha * g) * (1.0 + p->beta);",
     [("test_plain_expert_equals_textbook_ffn", dict(act="silu", alpha=1.702))]),
    ("unfused gate read from the up stack",
     "g += weight(p->gate, p->gate_scales, wdt, ee, F, d, f, i) * z[i];",
     "g += weight(gu, gus, wdt, ee, F, d, f, i) * z[i];",
     [("test_unfused_gate_stack_equals_concat", {})]),
    ("router weight read expert-major ([E, d])",
     "load(p->router_weight, p->act_dtype, i * E + e);",
     "load(p->router_weight, p->act_dtype, e * p->d + i);",
     [("test_router_weight_worked_example", {}), ("test_router_weight_matches_numpy_matmul", {})]),
    ("SiLU limit not applied to the up value",
     "u = u < p->limit ? (u > -p->limit ? u : -p->limit) : p->limit;",
     ";",
     [("test_single_expert_equals_textbook_ffn",
       dict(act="silu", alpha=1.702, beta=0.0, limit=0.5))]),
    ("kept weights renormalized with renormalize off (a softmax over the kept experts)",
     "if (p->renormalize) {",
     "if (1) {",
     [("test_softmax_without_renormalize_keeps_at_least_k_over_E", {}), ("test_routing_worked_example", {})]),
    ("e8m0 exponent bias 126",
     "return ldexp(1.0, s - 127);",
     "return ldexp(1.0, s - 126);",
     [("test_e8m0_table", {})]),
    ("e2m1 exponent bias 0",
     "ldexp(1.0 + 0.5 * m, ex - 1)",
     "ldexp(1.0 + 0.5 * m, ex)",
     [("test_e2m1_table", {})]),
    ("groups taken worst first",
     "outranks(gscore[g], g, gscore[best], best)",
     "outranks(gscore[best], best, gscore[g], g)",
     [("test_group_limited_selection_matches_exhaustive_search", dict(sel_std=0.0)),
      ("test_biased_group_selection_matches_exhaustive_search_on_independent_keys",
       dict(score="sigmoid"))]),
    ("sigmoid with the sign of its argument flipped",
     "static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }",
     "static double sigmoid(double v) { return 1.0 / (1.0 + exp(v)); }",
     [("test_softmax_and_sigmoid_scores_match_scipy", {}),
      ("test_single_expert_equals_textbook_ffn", dict(act="silu", alpha=1.0, beta=0.0, limit=0.0))]),
    ("GELU tanh form with a wrong cubic coefficient",
     "(g + 0.044715 * g * g * g)));\n    break;",
     "(g + 0.0447 * g * g * g)));\n    break;",
     [("test_single_expert_equals_textbook_ffn", dict(act="gelu_tanh", alpha=1.0, beta=0.0, limit=0.0))]),
    ("GELU erf form with its argument scaled by sqrt(2) instead of 1/sqrt(2)",
     "a = 0.5 * g * (1.0 + erf(g / sqrt(2.0))); break;",
     "a = 0.5 * g * (1.0 + erf(g * sqrt(2.0))); break;",
     [("test_single_expert_equals_textbook_ffn", dict(act="gelu_erf", alpha=1.0, beta=0.5, limit=0.0))]),
    ("shared expert weighed by the first routed weight",
     "for (int64_t i = 0; i < d; i++) y[i] += gate * o[i];",
     "for (int64_t i = 0; i < d; i++) y[i] += gate * w[0] * o[i];",
     [("test_shared_expert_with_sigmoid_gate", {})]),
    ("down stack read transposed ([F, d] per expert)",
     "acc += weight(dn, dns, wdt, ee, d, F, o, f) * h[f];",
     "acc += weight(dn, dns, wdt, ee, F, d, f, o) * h[f];",
     [("test_single_expert_equals_textbook_ffn", dict(act="relu", alpha=1.0, beta=0.0, limit=0.0))]),
]


def _compile(src_text, out_path):
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", out_path,
                    "-x", "c", "-", "-lm"], input=src_text.encode(), check=True)


@pytest.mark.parametrize("name,old,new,checks", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_a_planted_mistake(name, old, new, checks, tmp_path, monkeypatch):
    with open(oracle._SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    so = os.path.join(str(tmp_path), "libmoe_oracle_mutant.so")
    _compile(src.replace(old, new), so)
    monkeypatch.setattr(oracle, "_lib", oracle._bind(C.CDLL(so)))
    caught = []
    for fn, kwargs in checks:
        try:
            getattr(pins, fn)(None, **kwargs)
        except AssertionError:
            caught.append(fn)
    assert caught, f"no pin notices the planted mistake: {name}"


def test_unmodified_source_passes_the_same_pins(tmp_path, monkeypatch):
    """The harness itself: the unmodified source compiled the same way passes every check."""
    with open(oracle._SRC) as f:
        src = f.read()
    so = os.path.join(str(tmp_path), "libmoe_oracle_copy.so")
    _compile(src, so)
    monkeypatch.setattr(oracle, "_lib", oracle._bind(C.CDLL(so)))
    for _, _, _, checks in MUTATIONS:
        for fn, kwargs in checks:
            getattr(pins, fn)(None, **kwargs)
