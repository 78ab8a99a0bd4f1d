"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Sizes span several GEMM tiles with ragged tails in every dimension; each case
compares the routing bit-exactly and every output element within the
tolerance (1e-4 relative for fp32, 2e-2 for bf16, of max|y|).
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, make_inputs, small

from gpu_cases import check_output, check_routing, host, parity, run_gpu

pytestmark = pytest.mark.gpu

MIX = small(CONFIGS["mixtral_bf16"], name="mixtral_small", T=300, d=256, F=384)
DSK = small(CONFIGS["deepseek_bf16"], name="deepseek_small", T=130, d=256, F=128, E=64, k=8, Fs=192)
GPT = small(CONFIGS["gptoss_mxfp4"], name="gptoss_bf16_small", w_dtype="bf16", T=200, d=320, F=352,
            E=8, k=4)
DEC = small(CONFIGS["decode_T1"], name="decode_small", d=512, F=256, E=32)
FP4 = small(CONFIGS["gptoss_mxfp4"], name="gptoss_mxfp4_small", T=200, d=320, F=352, E=8, k=4)
TINY = CONFIGS["tiny_fp32"]

CASES = {
    "tiny_fp32": TINY,
    "tiny_fp32_options": small(TINY, name="tiny_fp32_options", gu_layout="interleaved", expert_bias=True,
                               router_bias=True, Fs=64, shared_gate=True, shared_output=True,
                               score="sigmoid", selection_bias_std=0.1, routed_scale=1.5),
    "mixtral_small": MIX,
    "deepseek_small": DSK,
    "gptoss_bf16_small": GPT,
    "decode_small_T1": DEC,
    "decode_small_T5": small(DEC, name="decode_small_T5", T=5),
    "shared_gate_and_output": small(DSK, name="shared_gate_and_output", shared_gate=True, shared_output=True),
    "weigh_inputs": small(MIX, name="weigh_inputs", weigh_inputs=True, renormalize=False),
    "no_renorm": small(MIX, name="no_renorm", renormalize=False, E=16, k=4),
    "gelu_erf": small(MIX, name="gelu_erf", act="gelu_erf", beta=0.5),
    "gelu_tanh": small(MIX, name="gelu_tanh", act="gelu_tanh"),
    "relu": small(MIX, name="relu", act="relu", expert_bias=True),
    "identity": small(MIX, name="identity", act="identity", beta=0.25),
    "f32_logits": small(MIX, name="f32_logits", logit_dtype="f32", router_bias=True),
    "T1": small(MIX, name="T1", T=1),
    "T3": small(MIX, name="T3", T=3),
    "T17": small(MIX, name="T17", T=17),
    "E5": small(MIX, name="E5", E=5, k=3),
    "E37": small(MIX, name="E37", E=37, k=3, T=90),
    "mostly_empty_experts": small(MIX, name="mostly_empty_experts", E=64, k=2, T=3),
    "k1": small(MIX, name="k1", k=1),
    "k_equals_E": small(MIX, name="k_equals_E", E=4, k=4, renormalize=False),
    "ragged_d_F": small(MIX, name="ragged_d_F", d=72, F=40, Fs=24, T=70),
    "many_experts": small(MIX, name="many_experts", E=256, k=8, T=64, d=128, F=64),
    "tiny_batch_shared_expert": small(DSK, name="tiny_batch_shared_expert", T=4, shared_gate=True,
                                      expert_bias=True),
    "tiny_batch_interleaved": small(MIX, name="tiny_batch_interleaved", T=8, gu_layout="interleaved",
                                    act="gelu_tanh", expert_bias=True, weigh_inputs=True),
    "gptoss_mxfp4_small": FP4,
    "mxfp4_concat": small(FP4, name="mxfp4_concat", gu_layout="concat", limit=0.0, alpha=1.0),
    "mxfp4_T1_many_experts": small(FP4, name="mxfp4_T1_many_experts", T=1, E=32, k=4),
    "mxfp4_big_rows": small(FP4, name="mxfp4_big_rows", T=700, E=4, k=2, d=256, F=256),
    # 450 rows per expert: a full 256-row tile and a 194-row one
    "mxfp4_three_row_tiles": small(FP4, name="mxfp4_three_row_tiles", T=450, E=2, k=2, d=256, F=256),
    # small batch over many experts with a long K (32-row activation tiles)
    "small_batch_long_k": small(CONFIGS["decode_T8"], name="small_batch_long_k", T=16, d=2048, F=384),
}


@pytest.mark.parametrize("name", list(CASES))
def test_forward_matches_oracle(name):
    parity(CASES[name])


@pytest.mark.parametrize("E,k,G,TG", [(64, 8, 8, 4), (32, 4, 4, 2), (40, 6, 5, 3), (256, 8, 8, 4)])
def test_routing_with_ties_and_groups(E, k, G, TG):
    # bf16 logits on a coarse grid produce many exact ties in keys and group scores
    cfg = small(DSK, name="route_ties", E=E, k=k, n_group=G, topk_group=TG, T=257, score="sigmoid",
                selection_bias_std=0.0)
    g = torch.Generator().manual_seed(E + k)
    logits = (torch.randint(-4, 5, (cfg.T, E), generator=g).float() * 0.25).to(torch.bfloat16)
    import mixture_experts_ffn_10_b200 as m
    inputs = {"logits": logits.cuda()}
    idx, w = m.route(cfg, inputs)
    torch.cuda.synchronize()
    check_routing(oracle.Problem(cfg, host(inputs)), idx, w)


@pytest.mark.parametrize("score,sel,groups", [("softmax", 0.0, 0), ("softmax", 0.05, 0), ("sigmoid", 0.1, 0),
                                              ("softmax", 0.05, 8), ("softmax", 0.1, 12)])
def test_routing_scores(score, sel, groups):
    # softmax with a selection bias ranks by softmax(l') + B ("Struct MoeSpec" selection_bias),
    # with and without a group limit
    cfg = small(MIX, name="route_scores", E=96, k=6, T=513, score=score, selection_bias_std=sel,
                router_bias=True, renormalize=score == "sigmoid", routed_scale=2.5,
                n_group=groups, topk_group=groups // 2)
    import mixture_experts_ffn_10_b200 as m
    inputs = make_inputs(cfg, "cuda", with_weights=False)
    idx, w = m.route(cfg, inputs)
    torch.cuda.synchronize()
    check_routing(oracle.Problem(cfg, host(inputs)), idx, w)


def test_renormalize_clamp_on_gpu():
    cfg = small(MIX, name="clamp", E=16, k=4, T=4, score="sigmoid")
    logits = torch.full((4, 16), -20.0).to(torch.bfloat16)
    import mixture_experts_ffn_10_b200 as m
    inputs = {"logits": logits.cuda()}
    idx, w = m.route(cfg, inputs)
    torch.cuda.synchronize()
    check_routing(oracle.Problem(cfg, host(inputs)), idx, w)


@pytest.mark.parametrize("cfg", [MIX, TINY], ids=["bf16", "f32"])
def test_bitwise_deterministic(cfg):
    inputs = make_inputs(cfg, "cuda")
    y1, i1, w1 = run_gpu(cfg, inputs)
    y2, i2, w2 = run_gpu(cfg, inputs)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(i1, i2) and torch.equal(w1, w2)


@pytest.mark.parametrize("cfg", [MIX, small(TINY, Fs=32)], ids=["bf16", "f32"])
def test_interleaved_layout_is_bitwise_equal_to_concat(cfg):
    inputs = make_inputs(cfg, "cuda")
    y1, _, _ = run_gpu(cfg, inputs)
    F = cfg.F
    perm = torch.stack([torch.arange(F), torch.arange(F) + F], 1).reshape(-1).cuda()
    il = dict(inputs)
    il["gate_up"] = inputs["gate_up"][:, perm].contiguous()
    if cfg.Fs:
        Fs = cfg.Fs
        ps = torch.stack([torch.arange(Fs), torch.arange(Fs) + Fs], 1).reshape(-1).cuda()
        il["shared_gate_up"] = inputs["shared_gate_up"][ps].contiguous()
    y2, _, _ = run_gpu(small(cfg, gu_layout="interleaved"), il)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_routed_scale_on_gpu():
    base = small(MIX, score="sigmoid", renormalize=True)
    inputs = make_inputs(base, "cuda")
    y1, _, _ = run_gpu(base, inputs)
    y2, _, _ = run_gpu(small(base, routed_scale=2.0), inputs)
    torch.cuda.synchronize()
    # scaling by a power of two is exact through every bf16 rounding step
    assert torch.equal(y2.float(), 2.0 * y1.float())


def test_shared_output_added_on_gpu():
    cfg = small(MIX, shared_output=True)
    inputs = make_inputs(cfg, "cuda")
    y, _, _ = run_gpu(cfg, inputs)
    p = oracle.Problem(cfg, host(inputs))
    torch.cuda.synchronize()
    check_output(cfg, y, p.forward(), "shared_output")


def test_zero_tokens_no_op_on_gpu():
    import mixture_experts_ffn_10_b200 as m
    cfg = small(MIX, T=0)
    inputs = make_inputs(cfg, "cuda")
    y = m.forward(cfg, inputs)
    torch.cuda.synchronize()
    assert y.shape == (0, cfg.d)


def _dequant_mxfp4(q, s):
    """bf16 weights equal to an MXFP4 stack, decoded with the oracle's own e2m1/e8m0 decoders."""
    table = torch.tensor([oracle.decode_e2m1(c) for c in range(16)], dtype=torch.float64)
    q = q.cpu().to(torch.int64)
    codes = torch.stack([q & 0xF, q >> 4], -1).reshape(*q.shape[:-1], q.shape[-1] * 2)
    scale = torch.tensor([oracle.decode_e8m0(v) for v in range(256)], dtype=torch.float64)[s.cpu().to(torch.int64)]
    w = table[codes] * scale.repeat_interleave(32, -1)
    out = w.to(torch.bfloat16)
    assert torch.equal(out.double(), w)  # every MXFP4 value is exact in bf16
    return out


@pytest.mark.parametrize("layout", ["interleaved", "concat"])
def test_mxfp4_path_equals_bf16_path_on_dequantized_weights(layout):
    cfg = small(FP4, gu_layout=layout)
    inputs = make_inputs(cfg, "cuda")
    y4, i4, _ = run_gpu(cfg, inputs)
    deq = dict(inputs)
    deq["gate_up"] = _dequant_mxfp4(inputs["gate_up"], inputs["gate_up_scales"]).cuda()
    deq["down"] = _dequant_mxfp4(inputs["down"], inputs["down_scales"]).cuda()
    deq["gate_up_scales"] = deq["down_scales"] = None
    yb, ib, _ = run_gpu(small(cfg, w_dtype="bf16"), deq)
    torch.cuda.synchronize()
    assert torch.equal(i4, ib)
    a, b = y4.float(), yb.float()
    assert (a - b).abs().max().item() <= 1e-2 * b.abs().max().item()


@pytest.mark.parametrize("cfg", [MIX, FP4, small(DSK, shared_gate=True)], ids=["bf16", "mxfp4", "shared"])
def test_forward_captured_in_a_cuda_graph_matches_eager(cfg):
    import mixture_experts_ffn_10_b200 as m
    inputs = make_inputs(cfg, "cuda")
    shape, opts = m.shape_of(cfg), m.options_of(cfg)
    ws = m.Workspace(m.moe_workspace_size(shape, opts))
    y = torch.empty_like(inputs["x"])
    tens = m.tensors_of(inputs, y)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):  # warm-up call outside the capture
        assert m.moe_forward(shape, opts, tens, ws.ptr, ws.nbytes, s.cuda_stream) == 0
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        assert m.moe_forward(shape, opts, tens, ws.ptr, ws.nbytes, s.cuda_stream) == 0
    # new inputs in the same buffers, then replay
    other = make_inputs(small(cfg, seed=cfg.seed + 77), "cuda", with_weights=False)
    inputs["x"].copy_(other["x"])
    inputs["logits"].copy_(other["logits"])
    g.replay()
    torch.cuda.synchronize()
    y_graph = y.clone()
    y_eager = m.forward(cfg, inputs)
    torch.cuda.synchronize()
    assert torch.equal(y_graph, y_eager)
    del g


def test_stage_events_inside_a_cuda_graph_time_every_replay():
    """moe_forward_events under stream capture: the events become graph nodes, each
    replay times the stages, and the output equals moe_forward's."""
    import mixture_experts_ffn_10_b200 as m
    cfg = MIX
    inputs = make_inputs(cfg, "cuda")
    shape, opts = m.shape_of(cfg), m.options_of(cfg)
    ws = m.Workspace(m.moe_workspace_size(shape, opts))
    y = torch.empty_like(inputs["x"])
    tens = m.tensors_of(inputs, y)
    s = torch.cuda.Stream()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(m.MOE_STAGE_EVENTS)]
    for ev in evs:
        ev.record(s)
    handles = [ev.cuda_event for ev in evs]
    with torch.cuda.stream(s):
        assert m.moe_forward(shape, opts, tens, ws.ptr, ws.nbytes, s.cuda_stream) == 0
    torch.cuda.synchronize()
    y_plain = y.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        assert m.moe_forward_events(shape, opts, tens, ws.ptr, ws.nbytes, s.cuda_stream, handles) == 0
    for _ in range(2):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_plain)
        stages = [evs[i].elapsed_time(evs[i + 1]) for i in range(len(evs) - 1)]
        assert all(t >= 0.0 for t in stages) and sum(stages) > 0.0
    del g


# The library's limits: E = 1024 experts (32 per routing lane), k = 32, 32 groups.
MAX_CASES = {
    "max_experts": small(MIX, name="max_experts", E=1024, k=8, T=64, d=128, F=64),
    "max_k": small(MIX, name="max_k", E=64, k=32, T=40, d=128, F=64, renormalize=True),
}


@pytest.mark.parametrize("name", list(MAX_CASES))
def test_maximum_sizes_match_oracle(name):
    parity(MAX_CASES[name])


def test_routing_with_the_maximum_group_count():
    cfg = small(DSK, name="max_groups", E=1024, k=8, n_group=32, topk_group=4, T=97, score="sigmoid",
                selection_bias_std=0.1)
    import mixture_experts_ffn_10_b200 as m
    inputs = make_inputs(cfg, "cuda", with_weights=False)
    idx, w = m.route(cfg, inputs)
    torch.cuda.synchronize()
    check_routing(oracle.Problem(cfg, host(inputs)), idx, w)


def test_routing_with_nan_and_infinite_logits():
    """NaN keys rank below every number (ties to the lower index); sigmoid(+inf) = 1 and
    sigmoid(-inf) = 0 are ordinary keys.  Token 0 has only NaN logits (its weights are
    NaN on both sides), token 1 only -inf and one NaN (weights 0 after the clamp)."""
    cfg = small(MIX, name="route_nonfinite", E=32, k=4, T=65, score="sigmoid", renormalize=True)
    g = torch.Generator().manual_seed(7)
    logits = torch.randn(cfg.T, cfg.E, generator=g)
    logits[torch.rand(cfg.T, cfg.E, generator=g) < 0.10] = float("nan")
    logits[torch.rand(cfg.T, cfg.E, generator=g) < 0.05] = float("inf")
    logits[torch.rand(cfg.T, cfg.E, generator=g) < 0.05] = float("-inf")
    logits[0] = float("nan")
    logits[1, :] = float("-inf")
    logits[1, 5] = float("nan")
    logits = logits.to(torch.bfloat16)
    import mixture_experts_ffn_10_b200 as m
    inputs = {"logits": logits.cuda()}
    idx, w = m.route(cfg, inputs)
    torch.cuda.synchronize()
    p = oracle.Problem(cfg, host(inputs))
    ri, rw, _, _ = p.route(0)
    assert np.array_equal(idx[0].cpu().numpy(), ri) and np.isnan(rw).all() and torch.isnan(w[0]).all()
    check_routing(p, idx, w, tokens=range(1, cfg.T))


def test_every_token_on_the_same_two_experts():
    """Extreme skew: experts 3 and 5 take all 600 tokens (five 128-row tiles each, a
    ragged last one), the other six experts are empty."""
    cfg = small(MIX, name="two_hot_experts", T=600, E=8, k=2)
    g = torch.Generator().manual_seed(11)
    logits = torch.randn(cfg.T, cfg.E, generator=g) * 0.1
    logits[:, 3] += 4.0
    logits[:, 5] += 3.0
    parity(cfg, override={"logits": logits.to(torch.bfloat16)})


@pytest.mark.parametrize("cfg", [DSK, MIX, small(DEC, T=5)], ids=["deepseek", "mixtral", "decode"])
def test_expert_visiting_order_does_not_change_results(cfg, monkeypatch):
    """The GEMMs' interleaved expert order (largest first, alternating with the
    smallest) only reorders independent tiles: results are bitwise those of the
    expert order."""
    inputs = make_inputs(cfg, "cuda")
    monkeypatch.setenv("MOE_B200_INTERLEAVE", "0")
    y0, i0, _ = run_gpu(cfg, inputs)
    monkeypatch.setenv("MOE_B200_INTERLEAVE", "1")
    y1, i1, _ = run_gpu(cfg, inputs)
    torch.cuda.synchronize()
    assert torch.equal(i0, i1) and torch.equal(y0, y1)
