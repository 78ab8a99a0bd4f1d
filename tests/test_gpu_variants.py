"""GPU parity of the layout and router variants (through the C ABI, against the oracle).

  - unfused gate stack ("MoE" set_weights gate_experts + gate_bias; graph-op fc3):
    every kernel family (single-CTA and CTA-pair bf16, MXFP4, fp32, split-K);
  - plain, non-gated experts (graph-op fc1 with fusion_size 1, activation_type relu /
    gelu / silu / identity), with and without a shared expert;
  - the router in front of the routing ("Struct MoeSpec" wr [d, E] and router_bias):
    routing bit-exact on every token, the logits it reports equal to the oracle's.
Outputs within the parity tolerance (1e-4 of max|y| for fp32, 2e-2 for bf16/MXFP4).
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, make_inputs, small

from gpu_cases import check_output, check_routing, host, parity, run_gpu

pytestmark = pytest.mark.gpu

MIX = small(CONFIGS["mixtral_bf16"], name="v_mixtral", T=300, d=256, F=384)
DSK = small(CONFIGS["deepseek_bf16"], name="v_deepseek", T=130, d=256, F=128, E=64, k=8, Fs=192)
DEC = small(CONFIGS["decode_T1"], name="v_decode", d=512, F=256, E=32)
FP4 = small(CONFIGS["gptoss_mxfp4"], name="v_mxfp4", T=200, d=320, F=352, E=8, k=4)
TINY = CONFIGS["tiny_fp32"]

CASES = {
    "unfused": small(MIX, name="unfused", gu_layout="unfused", expert_bias=True),
    "unfused_shared_gate": small(DSK, name="unfused_shared_gate", gu_layout="unfused", shared_gate=True,
                                 expert_bias=True),
    "unfused_T1_split_k": small(DEC, name="unfused_T1_split_k", gu_layout="unfused", expert_bias=True),
    "unfused_mxfp4": small(FP4, name="unfused_mxfp4", gu_layout="unfused"),
    "unfused_fp32": small(TINY, name="unfused_fp32", gu_layout="unfused", expert_bias=True, Fs=64),
    "plain_relu": small(MIX, name="plain_relu", ffn="plain", act="relu", expert_bias=True),
    "plain_silu_shared": small(DSK, name="plain_silu_shared", ffn="plain", act="silu", alpha=1.702,
                               shared_gate=True),
    "plain_gelu_T1_split_k": small(DEC, name="plain_gelu_T1_split_k", ffn="plain", act="gelu_tanh",
                                   expert_bias=True),
    "plain_identity_ragged": small(MIX, name="plain_identity_ragged", ffn="plain", act="identity",
                                   d=72, F=40, T=70),
    "plain_mxfp4": small(FP4, name="plain_mxfp4", ffn="plain", act="relu"),
    "plain_fp32": small(TINY, name="plain_fp32", ffn="plain", act="gelu_erf", Fs=64, expert_bias=True),
    "router_mixtral": small(MIX, name="router_mixtral", router="weight"),
    "router_deepseek": small(DSK, name="router_deepseek", router="weight", router_bias=True,
                             logit_dtype="f32"),
    "router_fp32": small(TINY, name="router_fp32", router="weight", score="sigmoid", renormalize=True),
    "router_mxfp4": small(FP4, name="router_mxfp4", router="weight"),
    "router_many_experts": small(MIX, name="router_many_experts", router="weight", E=300, k=6, T=77,
                                 d=136, F=64),
    # a shared expert (bf16 weights) beside MXFP4 routed experts ("ClikaRT::nn::QMoEWoQ"
    # forward with a shared branch; "Struct Moe" shared experts with any expert dtype)
    "mxfp4_shared_gate": small(FP4, name="mxfp4_shared_gate", Fs=192, shared_gate=True),
    "mxfp4_shared_plain": small(FP4, name="mxfp4_shared_plain", Fs=160, ffn="plain", act="relu"),
    "mxfp4_shared_T3": small(FP4, name="mxfp4_shared_T3", Fs=96, T=3),
}


@pytest.mark.parametrize("name", list(CASES))
def test_variant_matches_oracle(name, monkeypatch):
    if "split_k" in name:  # the split-K tensor-core GEMMs, not the few-token kernel
        monkeypatch.setenv("MOE_B200_GEMV", "0")
    parity(CASES[name])


@pytest.mark.parametrize("cfg", [MIX, small(DSK, Fs=0), FP4], ids=["bf16", "bf16_many", "mxfp4"])
def test_unfused_is_bitwise_equal_to_concat(cfg):
    """The same gate and up rows as one concatenated stack or two stacks: identical MMA
    operands, identical results."""
    inputs = make_inputs(small(cfg, gu_layout="unfused", expert_bias=True), "cuda")
    y_unf, _, _ = run_gpu(small(cfg, gu_layout="unfused", expert_bias=True), inputs)
    cat = dict(inputs)
    cat["gate_up"] = torch.cat([inputs["gate"], inputs["gate_up"]], 1).contiguous()
    if inputs["gate_scales"] is not None:
        cat["gate_up_scales"] = torch.cat([inputs["gate_scales"], inputs["gate_up_scales"]], 1).contiguous()
    cat["gate_up_bias"] = torch.cat([inputs["gate_bias"], inputs["gate_up_bias"]], 1).contiguous()
    cat["gate"] = cat["gate_scales"] = cat["gate_bias"] = None
    y_cat, _, _ = run_gpu(small(cfg, gu_layout="concat", expert_bias=True), cat)
    torch.cuda.synchronize()
    assert torch.equal(y_unf, y_cat)


def _router_logits_check(cfg, tokens=None):
    """Routing with the router weight: the reported logits equal the oracle's (bitwise:
    both sum x Wr in double in index order and round once), the routing bit-exact."""
    import mixture_experts_ffn_10_b200 as m
    inputs = make_inputs(cfg, "cuda", with_weights=False)
    shape, opts = m.shape_of(cfg), m.options_of(cfg)
    ws = m.Workspace(m.moe_workspace_size(shape, opts))
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    logits = torch.full((cfg.T, cfg.E), float("nan"), dtype=torch.float32, device="cuda")
    rc = m.moe_route(shape, opts, m.tensors_of(inputs, None, idx, w, logits), ws.ptr, ws.nbytes,
                     torch.cuda.current_stream().cuda_stream)
    assert rc == 0, m.moe_last_error()
    torch.cuda.synchronize()
    p = oracle.Problem(cfg, host(inputs))
    lg = logits.cpu().numpy()
    toks = range(cfg.T) if tokens is None else tokens
    # the oracle's logits: an unbiased softmax ranks by them, so its keys are the logits
    bare = dict(host(inputs), router_bias=None, selection_bias=None)
    plain = oracle.Problem(small(cfg, router_bias=False, selection_bias_std=0.0, score="softmax",
                                 n_group=0, topk_group=0), bare)
    for t in toks:
        _, _, keys, _ = plain.route(int(t))
        assert np.array_equal(lg[t].astype(np.float64), keys), f"token {t}: logits differ"
    check_routing(p, idx, w, tokens=toks)


@pytest.mark.parametrize("score,sel,groups", [("softmax", 0.0, 0), ("sigmoid", 0.1, 8), ("softmax", 0.05, 4)])
def test_router_weight_routing_is_bit_exact(score, sel, groups):
    cfg = small(DSK, name="router_route", T=257, d=384, E=64, k=6, router="weight", score=score,
                selection_bias_std=sel, n_group=groups, topk_group=groups // 2, router_bias=True)
    _router_logits_check(cfg)


FULL = ["mixtral_bf16", "gptoss_mxfp4", "deepseek_bf16", "decode_T1", "decode_T8", "decode_T64",
        "decode_T256", "tiny_fp32"]


@pytest.mark.parametrize("name", FULL)
def test_router_weight_routing_at_full_size(name):
    """The benchmark shapes with the router weight in place of the caller's logits:
    logits and routing of every token (a seeded sample of 512 for the 8192-token one)."""
    cfg = small(CONFIGS[name], router="weight")
    toks = None
    if cfg.T > 4096:
        toks = sorted(np.random.default_rng(cfg.seed).choice(cfg.T, 512, replace=False).tolist())
    _router_logits_check(cfg, toks)
