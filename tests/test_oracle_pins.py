"""Pins of the CPU oracle against facts fixed outside it (no GPU).

Each test checks the oracle against something other than itself: a value
derived by hand from the pages' definitions (tests/golden), a published format
table, a library routine (scipy / torch CPU), a brute-force search, or an
invariant the pages state.  Sources, by page title and item:
  "Struct MoeSpec": renormalize, score, selection_bias, groups, scale,
      weigh_inputs, sum_can_clamp;
  "Struct Moe": groups (two best experts), shared_gate;
  "MoE" graph-op page: fc1/fc2 layouts, swiglu_fusion, activation_alpha/beta,
      swiglu_limit, k;
  "ClikaRT::nn::QMoEWoQ": forward(..., shared_output) folded into the combine.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special as sp
import torch
import torch.nn.functional as Fn

import oracle
from workloads import MoeConfig, make_inputs, quantize_mxfp4, small

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _f32(v):
    return float(np.float32(v))


# ------------------------------------------------------------------ decoders


def test_e2m1_table(oracle_lib):
    for code, val in _rows("e2m1_codes.txt"):
        got = oracle.decode_e2m1(int(code))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_e8m0_table(oracle_lib):
    for s, val in _rows("e8m0_scales.txt"):
        got = oracle.decode_e8m0(int(s))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val)


def test_bf16_decoder_matches_torch_on_every_pattern(oracle_lib):
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.decode_bf16(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ------------------------------------------------------------------ MXFP4 encoding (input side)


def _dequant(q, s):
    """Plain MXFP4 dequantization with the spec table (tests/golden/e2m1_codes.txt)."""
    table = np.array([float(v) for _, v in _rows("e2m1_codes.txt")])
    q = q.numpy().astype(np.int64)
    codes = np.stack([q & 0xF, q >> 4], -1).reshape(*q.shape[:-1], q.shape[-1] * 2)
    scale = np.ldexp(1.0, s.numpy().astype(np.int64) - 127)
    return table[codes] * np.repeat(scale, 32, axis=-1)


def test_mxfp4_nibble_order_and_scale_by_hand():
    # one block of 32: value 6*2^-3 at k=0, -0.5*2^-3 at k=1, 1*2^-3 at k=2, rest 0.
    w = torch.zeros(1, 32)
    w[0, 0], w[0, 1], w[0, 2] = 0.75, -0.0625, 0.125
    q, s = quantize_mxfp4(w)
    # amax 0.75 -> floor(log2 .75) = -1 -> s = -1 - 2 + 127 = 124 (scale 2^-3)
    assert s.tolist() == [[124]]
    # codes: 6.0 -> 7, -0.5 -> 8|1 = 9, 1.0 -> 2; low nibble = even element
    assert q[0, 0].item() == (9 << 4) | 7
    assert q[0, 1].item() == 2


def test_mxfp4_exact_roundtrip_for_representable_values():
    g = torch.Generator().manual_seed(7)
    grid = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6])
    codes = torch.randint(0, 8, (64, 128), generator=g)
    sign = torch.randint(0, 2, (64, 128), generator=g) * 2 - 1
    exps = torch.randint(-10, 4, (64, 4), generator=g).repeat_interleave(32, 1)
    w = grid[codes] * sign * torch.pow(2.0, exps.float())
    w[:, ::32] = 6.0 * torch.pow(2.0, exps[:, ::32].float())   # pin each block's amax to 6*2^e
    q, s = quantize_mxfp4(w)
    assert np.array_equal(_dequant(q, s), w.double().numpy())


def test_mxfp4_rounding_error_bound():
    g = torch.Generator().manual_seed(8)
    w = torch.randn(32, 256, generator=g) * 0.02
    q, s = quantize_mxfp4(w)
    dq = _dequant(q, s)
    scale = np.repeat(np.ldexp(1.0, s.numpy().astype(np.int64) - 127), 32, -1)
    a = np.abs(w.double().numpy()) / scale
    err = np.abs(dq - w.double().numpy()) / scale
    # nearest-value rounding: error <= half the grid spacing around the value
    half = np.where(a <= 2, 0.25, np.where(a <= 4, 0.5, 1.0))
    inside = a <= 6
    assert (err[inside] <= half[inside] + 1e-12).all()
    # values in (6, 8) units saturate to +-6 (the scale puts amax in [4, 8) units)
    assert (a < 8).all() and np.array_equal(np.abs(dq[~inside]) / scale[~inside], np.full((~inside).sum(), 6.0))


# ------------------------------------------------------------------ routing


def _cfg(**kw):
    base = dict(name="pin", T=16, d=32, F=32, E=8, k=2, act_dtype="f32", w_dtype="f32",
                logit_dtype="f32", seed=77)
    base.update(kw)
    return MoeConfig(**base)


def _problem(cfg, **over):
    t = make_inputs(cfg, "cpu")
    t.update(over)
    return oracle.Problem(cfg, t), t


def test_routing_worked_example(oracle_lib):
    logits = torch.log(torch.arange(1, 5, dtype=torch.float32)).reshape(1, 4)
    for case, renorm, scale, w0, w1 in _rows("routing_worked_example.txt"):
        cfg = _cfg(T=1, E=4, k=2, renormalize=bool(int(renorm)), routed_scale=float(scale))
        p, _ = _problem(cfg, logits=logits)
        idx, w, _, _ = p.route(0)
        assert idx.tolist() == [3, 2], case
        assert np.allclose(w, [float(w0), float(w1)], rtol=1e-6, atol=0), case


def _best_subset(keys, cand, k):
    """Brute force: the k-subset of ``cand`` whose (key desc, index asc) ranking is best."""
    def rank_tuple(sub):
        return sorted(((-keys[e], e) for e in sub))
    best = min(itertools.combinations(cand, k), key=rank_tuple)
    return [e for _, e in rank_tuple(best)]


@pytest.mark.parametrize("E,k", [(1, 1), (3, 3), (6, 2), (8, 3), (10, 4), (12, 1)])
def test_topk_matches_brute_force_with_ties(oracle_lib, E, k):
    g = torch.Generator().manual_seed(E * 31 + k)
    # logits on a coarse grid: many exact ties exercise the lower-index rule
    logits = torch.randint(-2, 3, (40, E), generator=g).float() * 0.5
    cfg = _cfg(T=40, E=E, k=k)
    p, _ = _problem(cfg, logits=logits)
    for t in range(40):
        idx, _, keys, _ = p.route(t)
        assert idx.tolist() == _best_subset(keys, range(E), k)
        # the unbiased softmax ranks by the logit itself
        assert np.array_equal(keys, logits[t].double().numpy())


def test_softmax_and_sigmoid_scores_match_scipy(oracle_lib):
    for score in ("softmax", "sigmoid"):
        cfg = _cfg(T=8, E=16, k=4, score=score, router_bias=True, logit_dtype="bf16")
        p, t = _problem(cfg)
        lp = (t["logits"].float() + t["router_bias"].float()).double().numpy()  # fp32 add
        for tok in range(8):
            _, _, _, s = p.route(tok)
            ref = sp.softmax(lp[tok]) if score == "softmax" else sp.expit(lp[tok])
            assert np.allclose(s, ref, rtol=1e-13, atol=0)


def test_renormalized_weights_sum_to_one_times_scale(oracle_lib):
    for score, S in (("softmax", 1.0), ("sigmoid", 2.5)):
        cfg = _cfg(T=32, E=16, k=4, score=score, routed_scale=S)
        p, _ = _problem(cfg)
        _, w = p.route_all()
        assert np.allclose(w.sum(1), _f32(S), rtol=1e-12, atol=0)


def test_softmax_without_renormalize_keeps_at_least_k_over_E(oracle_lib):
    E, k = 16, 3
    cfg = _cfg(T=64, E=E, k=k, renormalize=False)
    p, t = _problem(cfg)
    idx, w = p.route_all()
    assert (w.sum(1) >= k / E - 1e-15).all()
    probs = sp.softmax(t["logits"].double().numpy(), axis=1)
    assert np.allclose(w, np.take_along_axis(probs, idx.astype(np.int64), 1), rtol=1e-13, atol=0)


def test_renormalize_clamp_binds_only_for_small_sigmoid_sums(oracle_lib):
    E, k = 8, 4
    logits = torch.full((2, E), -20.0)
    logits[1] = torch.linspace(-3, 3, E)
    cfg = _cfg(T=2, E=E, k=k, score="sigmoid")
    p, _ = _problem(cfg, logits=logits)
    _, w, _, s = p.route(0)
    kept = np.sort(sp.expit(logits[0].double().numpy()))[::-1][:k]
    assert kept.sum() < 2.0 ** -14
    assert np.allclose(w, kept / 2.0 ** -14, rtol=1e-13)
    _, w1, _, _ = p.route(1)
    assert abs(w1.sum() - 1.0) < 1e-12


def test_selection_bias_changes_choice_not_weight(oracle_lib):
    E, k = 16, 4
    cfg = _cfg(T=24, E=E, k=k, score="sigmoid", renormalize=False)
    p0, t = _problem(cfg)
    zero = torch.zeros(E)
    pz, _ = _problem(cfg, selection_bias=zero)
    big = torch.zeros(E)
    big[[1, 5]] = 10.0                       # forces experts 1 and 5 into every selection
    pb, _ = _problem(cfg, selection_bias=big)
    lp = t["logits"].double().numpy()
    for tok in range(24):
        i0, w0, _, _ = p0.route(tok)
        iz, wz, _, _ = pz.route(tok)
        assert np.array_equal(i0, iz) and np.array_equal(w0, wz)
        ib, wb, kb, _ = pb.route(tok)
        assert ib[0] in (1, 5) and ib[1] in (1, 5)
        # weight = the chosen expert's unbiased sigmoid, never the biased key
        assert np.allclose(wb, sp.expit(lp[tok][ib]), rtol=1e-13)
        assert ib.tolist() == _best_subset(kb, range(E), k)


def test_softmax_selection_bias_worked_example(oracle_lib):
    """"Struct MoeSpec" selection_bias on a softmax score: chosen by s + B, weighed by s.
    The fixture's numbers are chosen so that biasing the logit instead (l + B, or
    softmax(l + B), which ranks the same way) or ignoring B picks (3, 2), not (3, 0)."""
    logits = torch.log(torch.arange(1, 5, dtype=torch.float32)).reshape(1, 4)
    bias = torch.tensor([0.25, 0.125, 0.0, 0.0])
    for case, renorm, scale, i0, i1, w0, w1 in _rows("routing_selection_bias_example.txt"):
        cfg = _cfg(T=1, E=4, k=2, renormalize=bool(int(renorm)), routed_scale=float(scale))
        p, _ = _problem(cfg, logits=logits, selection_bias=bias)
        idx, w, keys, s = p.route(0)
        assert idx.tolist() == [int(i0), int(i1)], case
        assert np.allclose(w, [float(w0), float(w1)], rtol=1e-6, atol=0), case
        assert np.allclose(keys, [0.35, 0.325, 0.3, 0.4], rtol=1e-6, atol=0), case


def _independent_keys(lp, score, bias):
    """Selection keys computed here, outside the oracle: score(l') + B (scipy)."""
    s = sp.softmax(lp) if score == "softmax" else sp.expit(lp)
    return s, s + (bias if bias is not None else 0.0)


@pytest.mark.parametrize("score,E,k,renorm,S", [
    ("softmax", 6, 2, True, 1.0), ("softmax", 9, 3, False, 1.0), ("softmax", 12, 4, True, 2.5),
    ("sigmoid", 8, 3, True, 2.5), ("sigmoid", 11, 2, False, 1.0)])
def test_biased_selection_matches_brute_force_on_independent_keys(oracle_lib, score, E, k, renorm, S):
    """Random l' and B ~ N(0, 0.1): the chosen set is the best k-subset by
    (score(l') + B descending, index ascending) with the scores computed by scipy,
    and the weights are the unbiased scores of that set (renormalized, times S)."""
    T = 40
    cfg = _cfg(T=T, E=E, k=k, score=score, renormalize=renorm, routed_scale=S,
               selection_bias_std=0.1, router_bias=True)
    p, t = _problem(cfg)
    lp = (t["logits"].float() + t["router_bias"].float()).double().numpy()  # fp32 add
    bias = t["selection_bias"].double().numpy()
    for tok in range(T):
        s, key = _independent_keys(lp[tok], score, bias)
        want = _best_subset(key, range(E), k)
        idx, w, _, _ = p.route(tok)
        assert idx.tolist() == want, tok
        ws = s[want]
        if renorm:
            ws = ws / max(ws.sum(), 2.0 ** -14)
        assert np.allclose(w, ws * _f32(S), rtol=1e-12, atol=0), tok


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_biased_group_selection_matches_exhaustive_search_on_independent_keys(oracle_lib, score):
    """Groups on keys score(l') + B computed outside the oracle: a group scores the
    sum of its best two keys (any pair), the best topk_group groups are kept, then the
    best k experts among them."""
    E, G, TG, k = 12, 4, 2, 3
    per = E // G
    cfg = _cfg(T=40, E=E, k=k, score=score, n_group=G, topk_group=TG, selection_bias_std=0.1)
    p, t = _problem(cfg)
    lp = t["logits"].double().numpy()
    bias = t["selection_bias"].double().numpy()
    for tok in range(40):
        _, key = _independent_keys(lp[tok], score, bias)
        gs = [max(key[a] + key[b] for a, b in itertools.combinations(range(q * per, (q + 1) * per), 2))
              for q in range(G)]
        best_groups = min(itertools.combinations(range(G), TG),
                          key=lambda sub: sorted((-gs[q], q) for q in sub))
        cand = [e for q in sorted(best_groups) for e in range(q * per, (q + 1) * per)]
        idx, _, _, _ = p.route(tok)
        assert idx.tolist() == _best_subset(key, cand, k), tok


@pytest.mark.parametrize("sel_std", [0.0, 0.1])
def test_group_limited_selection_matches_exhaustive_search(oracle_lib, sel_std):
    E, G, TG, k = 16, 4, 2, 3
    per = E // G
    cfg = _cfg(T=48, E=E, k=k, score="sigmoid", n_group=G, topk_group=TG, selection_bias_std=sel_std)
    g = torch.Generator().manual_seed(5)
    logits = torch.randint(-3, 4, (48, E), generator=g).float() * 0.25   # ties in groups too
    p, _ = _problem(cfg, logits=logits)
    for tok in range(48):
        idx, _, keys, _ = p.route(tok)
        # group score: best pair sum, over every pair in the group
        gs = [max(keys[a] + keys[b] for a, b in itertools.combinations(range(q * per, (q + 1) * per), 2))
              for q in range(G)]
        best_groups = min(itertools.combinations(range(G), TG),
                          key=lambda sub: sorted((-gs[q], q) for q in sub))
        cand = [e for q in sorted(best_groups) for e in range(q * per, (q + 1) * per)]
        assert idx.tolist() == _best_subset(keys, cand, k)


def test_nan_key_ranks_last(oracle_lib):
    logits = torch.tensor([[float("nan"), -5.0, 0.0, float("-inf")]])
    cfg = _cfg(T=1, E=4, k=4, score="sigmoid")
    p, _ = _problem(cfg, logits=logits)
    idx, _, _, _ = p.route(0)
    assert idx.tolist() == [2, 1, 3, 0]


# ------------------------------------------------------------------ expert FFN and combine


def _dense_ffn(x, wg, wu, wd, act="silu", alpha=1.0, beta=0.0, limit=0.0, bg=None, bu=None, bd=None):
    """Textbook gated FFN with torch fp64 library activations."""
    g = x @ wg.T + (bg if bg is not None else 0)
    u = x @ wu.T + (bu if bu is not None else 0)
    if act == "silu":
        if limit > 0:
            g = torch.clamp(g, max=limit)
            u = torch.clamp(u, -limit, limit)
        a = g * torch.sigmoid(alpha * g)
    elif act == "gelu_erf":
        a = Fn.gelu(g, approximate="none")
    elif act == "gelu_tanh":
        a = Fn.gelu(g, approximate="tanh")
    elif act == "relu":
        a = Fn.relu(g)
    else:
        a = g
    return (a * (u + beta)) @ wd.T + (bd if bd is not None else 0)


def test_expert_worked_example(oracle_lib):
    for case, alpha, beta, y0, y1 in _rows("expert_worked_example.txt"):
        cfg = _cfg(T=1, d=2, F=1, E=1, k=1, alpha=float(alpha), beta=float(beta))
        x = torch.tensor([[1.0, 2.0]])
        gu = torch.tensor([[[1.0, 0.0], [0.0, 1.0]]])
        dn = torch.tensor([[[1.0], [0.5]]])
        p, _ = _problem(cfg, x=x, gate_up=gu, down=dn, logits=torch.zeros(1, 1))
        y = p.forward()[0]
        assert np.allclose(y, [float(y0), float(y1)], rtol=1e-15), case


@pytest.mark.parametrize("act,alpha,beta,limit", [
    ("silu", 1.0, 0.0, 0.0), ("silu", 1.702, 1.0, 7.0), ("silu", 1.702, 0.0, 0.5),
    ("gelu_erf", 1.0, 0.5, 0.0), ("gelu_tanh", 1.0, 0.0, 0.0), ("relu", 1.0, 0.0, 0.0),
    ("identity", 1.0, 0.25, 0.0)])
def test_single_expert_equals_textbook_ffn(oracle_lib, act, alpha, beta, limit):
    cfg = _cfg(T=6, d=24, F=40, E=1, k=1, act=act, alpha=alpha, beta=beta, limit=limit,
               expert_bias=True)
    t = make_inputs(cfg, "cpu")
    x32 = t["x"] * 3.0          # larger inputs so a small limit binds
    p, _ = _problem(cfg, x=x32)
    x = x32.double()
    F_ = cfg.F
    gu = t["gate_up"][0].double()
    b = t["gate_up_bias"][0].double()
    ref = _dense_ffn(x, gu[:F_], gu[F_:], t["down"][0].double(), act, _f32(alpha), _f32(beta),
                     _f32(limit), b[:F_], b[F_:], t["down_bias"][0].double())
    assert np.allclose(p.forward(), ref.numpy(), rtol=1e-12, atol=1e-12)
    if limit == 0.5:   # the clamp binds somewhere in this case
        g = x @ gu[:F_].T + b[:F_]
        assert (g > limit).any()


def test_interleaved_layout_equals_concat(oracle_lib):
    cfg = _cfg(T=10, d=32, F=24, E=4, k=2, expert_bias=True)
    p, t = _problem(cfg)
    F_ = cfg.F
    perm = torch.stack([torch.arange(F_), torch.arange(F_) + F_], 1).reshape(-1)  # g0,u0,g1,u1...
    pi, _ = _problem(small(cfg, gu_layout="interleaved"), gate_up=t["gate_up"][:, perm],
                     gate_up_bias=t["gate_up_bias"][:, perm])
    assert np.array_equal(p.forward(), pi.forward())


def test_k_equals_E_softmax_is_dense_mixture(oracle_lib):
    E = 5
    cfg = _cfg(T=7, d=16, F=12, E=E, k=E, renormalize=False)
    p, t = _problem(cfg)
    probs = sp.softmax(t["logits"].double().numpy(), axis=1)
    x = t["x"].double().numpy()
    y = p.forward()
    for tok in range(7):
        ref = sum(probs[tok, e] * p.expert(e, x[tok]) for e in range(E))
        assert np.allclose(y[tok], ref, rtol=1e-12, atol=1e-14)


def test_weigh_inputs_is_quadratic_for_identity_activation(oracle_lib):
    cfg = _cfg(T=9, d=16, F=8, E=6, k=3, act="identity")
    p, t = _problem(cfg)
    pw, _ = _problem(small(cfg, weigh_inputs=True))
    idx, w = p.route_all()
    x = t["x"].double().numpy()
    y = pw.forward()
    for tok in range(9):
        ref = sum(w[tok, j] ** 2 * p.expert(int(idx[tok, j]), x[tok]) for j in range(3))
        assert np.allclose(y[tok], ref, rtol=1e-12, atol=1e-14)


def test_routed_scale_is_linear(oracle_lib):
    cfg = _cfg(T=8, E=8, k=3, score="sigmoid")
    y1 = _problem(cfg)[0].forward()
    y25 = _problem(small(cfg, routed_scale=2.5))[0].forward()
    assert np.allclose(y25, 2.5 * y1, rtol=1e-13, atol=1e-15)


def test_shared_output_adds_exactly(oracle_lib):
    cfg = _cfg(T=8, E=4, k=2)
    p, t = _problem(cfg)
    z = torch.randn(8, cfg.d, generator=torch.Generator().manual_seed(3))
    pz, _ = _problem(small(cfg, shared_output=True), shared_output=z)
    assert np.allclose(pz.forward() - p.forward(), z.double().numpy(), rtol=0, atol=1e-13)


def test_shared_expert_with_sigmoid_gate(oracle_lib):
    cfg = _cfg(T=6, d=16, F=8, E=4, k=2, Fs=12, shared_gate=True)
    p, t = _problem(cfg)
    base = _problem(small(cfg, Fs=0, shared_gate=False))[0].forward()
    x = t["x"].double()
    sgu = t["shared_gate_up"].double()
    ffn = _dense_ffn(x, sgu[:12], sgu[12:], t["shared_down"].double())
    gate = torch.sigmoid(x @ t["shared_gate_vec"].double())
    assert np.allclose(p.forward() - base, (gate[:, None] * ffn).numpy(), rtol=1e-10, atol=1e-13)


def test_mxfp4_experts_equal_dequantized_experts(oracle_lib):
    cfg = _cfg(T=5, d=64, F=32, E=3, k=2, w_dtype="mxfp4", act_dtype="bf16", logit_dtype="bf16",
               gu_layout="interleaved", expert_bias=True)
    p, t = _problem(cfg)
    gu = torch.from_numpy(_dequant(t["gate_up"], t["gate_up_scales"])).float()
    dn = torch.from_numpy(_dequant(t["down"], t["down_scales"])).float()
    pd, _ = _problem(small(cfg, w_dtype="f32"), gate_up=gu, down=dn, gate_up_scales=None,
                     down_scales=None)
    assert np.array_equal(p.forward(), pd.forward())


def test_thread_count_does_not_change_results(oracle_lib):
    cfg = _cfg(T=12, E=8, k=2)
    p, _ = _problem(cfg)
    assert np.array_equal(p.forward(nthreads=1), p.forward(nthreads=4))


# ------------------------------------------------------------------ layouts, plain FFN, router weight


def test_unfused_gate_stack_equals_concat(oracle_lib):
    """Unfused ("MoE" set_weights gate_experts + gate_bias; graph-op fc3): the gate
    rows come from their own stack and gate_up holds the up rows.  Stacking gate on
    top of up gives the concatenated layout, which must give the same y."""
    cfg = _cfg(T=10, d=32, F=24, E=4, k=2, expert_bias=True, gu_layout="unfused", Fs=16)
    p, t = _problem(cfg)
    cat = torch.cat([t["gate"], t["gate_up"]], 1)
    cat_bias = torch.cat([t["gate_bias"], t["gate_up_bias"]], 1)
    pc, _ = _problem(small(cfg, gu_layout="concat"), gate_up=cat, gate_up_bias=cat_bias, gate=None,
                     gate_bias=None, shared_gate_up=t["shared_gate_up"], x=t["x"])
    assert np.array_equal(p.forward(), pc.forward())


def test_unfused_mxfp4_gate_stack_equals_concat(oracle_lib):
    cfg = _cfg(T=5, d=64, F=32, E=3, k=2, w_dtype="mxfp4", act_dtype="bf16", logit_dtype="bf16",
               gu_layout="unfused")
    p, t = _problem(cfg)
    pc, _ = _problem(small(cfg, gu_layout="concat"), gate_up=torch.cat([t["gate"], t["gate_up"]], 1),
                     gate_up_scales=torch.cat([t["gate_scales"], t["gate_up_scales"]], 1), gate=None,
                     gate_scales=None)
    assert np.array_equal(p.forward(), pc.forward())


def _plain_ffn(x, w1, wd, act, alpha, b1=None, bd=None):
    """Textbook non-gated FFN with torch fp64 library activations."""
    g = x @ w1.T + (b1 if b1 is not None else 0)
    if act == "silu":
        a = g * torch.sigmoid(alpha * g)
    elif act == "gelu_erf":
        a = Fn.gelu(g, approximate="none")
    elif act == "gelu_tanh":
        a = Fn.gelu(g, approximate="tanh")
    elif act == "relu":
        a = Fn.relu(g)
    else:
        a = g
    return a @ wd.T + (bd if bd is not None else 0)


@pytest.mark.parametrize("act,alpha", [("silu", 1.0), ("silu", 1.702), ("gelu_erf", 1.0),
                                       ("gelu_tanh", 1.0), ("relu", 1.0), ("identity", 1.0)])
def test_plain_expert_equals_textbook_ffn(oracle_lib, act, alpha):
    """Graph-op page "MoE": fc1 [E, fusion_size * inter, hidden] with fusion_size 1 and
    activation_type relu / gelu / silu / identity: h = act(fc1 x + b1), y = fc2 h + b2
    (beta and the SwiGLU limit do not apply: there is no up value)."""
    cfg = _cfg(T=6, d=24, F=40, E=1, k=1, ffn="plain", act=act, alpha=alpha, beta=0.75, limit=0.5,
               expert_bias=True)
    p, t = _problem(cfg)
    ref = _plain_ffn(t["x"].double(), t["gate_up"][0].double(), t["down"][0].double(), act, _f32(alpha),
                     t["gate_up_bias"][0].double(), t["down_bias"][0].double())
    assert np.allclose(p.forward(), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_plain_shared_expert(oracle_lib):
    cfg = _cfg(T=6, d=16, F=8, E=4, k=2, Fs=12, ffn="plain", act="relu")
    p, t = _problem(cfg)
    base = _problem(small(cfg, Fs=0))[0].forward()
    ffn = _plain_ffn(t["x"].double(), t["shared_gate_up"].double(), t["shared_down"].double(), "relu", 1.0)
    assert np.allclose(p.forward() - base, ffn.numpy(), rtol=1e-10, atol=1e-13)


def test_router_weight_worked_example(oracle_lib):
    x = torch.tensor([[1.0, 2.0, 3.0], [-1.0, 0.0, 2.0]])
    wr = torch.tensor([[1.0, 0.0], [0.0, 1.0], [1.0, -1.0]])
    cfg = _cfg(T=2, d=3, F=8, E=2, k=1, router="weight")
    p, _ = _problem(cfg, x=x, router_weight=wr)
    for tok, l0, l1 in _rows("router_worked_example.txt"):
        _, _, keys, _ = p.route(int(tok))
        assert keys.tolist() == [float(l0), float(l1)]   # unbiased softmax ranks by the logit


def test_router_weight_matches_numpy_matmul(oracle_lib):
    """Logits from Wr [d, E] equal numpy's fp64 x @ Wr rounded once to fp32 (to one fp32
    ulp: the two sums may round differently in the last double bit), and the routing
    on them equals the routing on those logits passed in."""
    cfg = _cfg(T=12, d=64, F=8, E=16, k=4, router="weight", act_dtype="bf16", w_dtype="bf16",
               router_bias=True, logit_dtype="f32")
    p, t = _problem(cfg)
    x = t["x"].double().numpy()
    wr = t["router_weight"].double().numpy()
    ref = (x @ wr).astype(np.float32)
    br = t["router_bias"].numpy()
    cfg_l = small(cfg, router="logits")
    pl, _ = _problem(cfg_l, logits=torch.from_numpy(ref), router_bias=t["router_bias"])
    for tok in range(cfg.T):
        _, _, keys, _ = p.route(tok)
        want = (ref[tok] + br).astype(np.float64)
        assert np.all(np.abs(keys - want) <= np.spacing(np.abs(want).astype(np.float32)).astype(np.float64))
        if np.array_equal(keys, want):
            assert np.array_equal(p.route(tok)[0], pl.route(tok)[0])
