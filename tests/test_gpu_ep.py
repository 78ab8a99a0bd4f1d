"""GPU checks of the expert-parallel building blocks and of the layer on one rank.

moe_permute against a host restatement of the sort (exact: indices, counts, weights,
rows); moe_experts_forward against the oracle's expert FFN row by row; moe_combine
against a sequential fp32 sum (bitwise); ExpertParallelMoE on one rank (the exchange is
a copy) against the oracle's forward and against moe_forward."""
import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, make_inputs, small

from gpu_cases import check_output, host

pytestmark = pytest.mark.gpu

DEC = small(CONFIGS["decode_T1"], name="ep_decode", T=40, d=256, F=128, E=16, k=4)
CASES = {
    "decode_small": DEC,
    "mixtral_small": small(CONFIGS["mixtral_bf16"], name="ep_mixtral", T=300, d=256, F=384),
    "unfused_bias_weigh_inputs": small(DEC, name="ep_unfused", gu_layout="unfused", expert_bias=True,
                                       weigh_inputs=True),
    "plain_relu": small(DEC, name="ep_plain", ffn="plain", act="relu", expert_bias=True),
    "fp32": small(CONFIGS["tiny_fp32"], name="ep_fp32", Fs=0),
    "mxfp4": small(CONFIGS["gptoss_mxfp4"], name="ep_mxfp4", T=100, d=320, F=352, E=8, k=4),
    # 64 routed rows: the expert forward reads its rows in place (one launch for both GEMMs)
    "rows_in_place": small(DEC, name="ep_in_place", T=16),
    # routed on x . router_weight (no logits given)
    "router_weight": small(DEC, name="ep_router", router="weight", router_bias=True),
}


def _m():
    import mixture_experts_ffn_10_b200 as m
    return m


@pytest.mark.parametrize("per_rank", [0, 4])
def test_permute_is_the_stable_expert_sort(per_rank):
    m = _m()
    from mixture_experts_ffn_10_b200.ep import LibraryOps
    cfg = CASES["decode_small"]
    inputs = make_inputs(cfg, "cuda")
    idx, w = m.route(cfg, inputs)
    x_perm, row_expert, row_w, counts, pos = LibraryOps().permute(cfg, idx, w, inputs["x"], per_rank)
    torch.cuda.synchronize()
    flat = idx.reshape(-1).cpu().numpy()
    order = np.argsort(flat, kind="stable")
    ref_pos = np.empty_like(order)
    ref_pos[order] = np.arange(order.size)
    e = flat[order]
    assert np.array_equal(counts.cpu().numpy(), np.bincount(flat, minlength=cfg.E))
    assert np.array_equal(pos.cpu().numpy().reshape(-1), ref_pos)
    assert np.array_equal(row_expert.cpu().numpy(), e % per_rank if per_rank else e)
    assert torch.equal(row_w.cpu(), w.reshape(-1).cpu()[torch.from_numpy(order)])
    assert torch.equal(x_perm.cpu(), inputs["x"].cpu()[torch.from_numpy(order // cfg.k)])


@pytest.mark.parametrize("rows", [50, 70])
@pytest.mark.parametrize("name", ["decode_small", "unfused_bias_weigh_inputs", "plain_relu", "fp32", "mxfp4"])
def test_experts_forward_matches_the_oracle_row_by_row(name, rows):
    from mixture_experts_ffn_10_b200.ep import LibraryOps, _with
    cfg = CASES[name]
    inputs = make_inputs(cfg, "cuda")
    g = torch.Generator().manual_seed(7)
    row_expert = torch.randint(0, cfg.E, (rows,), generator=g, dtype=torch.int32)
    row_w = torch.rand(rows, generator=g, dtype=torch.float32) + 0.25
    x = inputs["x"][torch.arange(rows) % cfg.T]
    cfg_rows = _with(cfg, T=rows, k=1, Fs=0, shared_gate=False)
    weights = {k: v for k, v in inputs.items() if k not in ("x", "logits", "router_weight", "shared_gate_up",
                                                            "shared_down", "shared_gate_vec", "shared_output")}
    y = LibraryOps().experts_forward(cfg_rows, x.contiguous(), row_expert.cuda(), row_w.cuda(), weights)
    torch.cuda.synchronize()
    p = oracle.Problem(cfg, host(inputs))
    xs = x.float().cpu().double().numpy()
    ref = np.stack([p.expert(int(e), float(wr) * xs[r]) if cfg.weigh_inputs else float(wr) * p.expert(int(e), xs[r])
                    for r, (e, wr) in enumerate(zip(row_expert.tolist(), row_w.tolist()))])
    check_output(cfg, y, ref, name)


def test_combine_sums_in_slot_order():
    from mixture_experts_ffn_10_b200.ep import LibraryOps
    cfg = CASES["decode_small"]
    g = torch.Generator().manual_seed(3)
    rows = cfg.T * cfg.k
    Y = torch.randn((rows, cfg.d), generator=g).to(torch.bfloat16)
    pos = torch.randperm(rows, generator=g).to(torch.int32).reshape(cfg.T, cfg.k)
    so = torch.randn((cfg.T, cfg.d), generator=g).to(torch.bfloat16)
    y = LibraryOps().combine(cfg, pos.cuda(), Y.cuda(), so.cuda())
    torch.cuda.synchronize()
    acc = torch.zeros((cfg.T, cfg.d), dtype=torch.float32)
    for j in range(cfg.k):
        acc = acc + Y[pos[:, j].long()].float()
    ref = (acc + so.float()).to(torch.bfloat16)
    assert torch.equal(y.cpu(), ref)


@pytest.mark.parametrize("name", list(CASES))
def test_layer_on_one_rank_matches_oracle_and_forward(name):
    m = _m()
    from mixture_experts_ffn_10_b200.ep import ExpertParallelMoE
    cfg = CASES[name]
    inputs = make_inputs(cfg, "cuda")
    local = {k: v for k, v in inputs.items() if k not in ("x", "logits")}
    y = ExpertParallelMoE(cfg, local).forward(inputs["x"], inputs.get("logits"))
    y_ref = m.forward(cfg, inputs)
    torch.cuda.synchronize()
    p = oracle.Problem(cfg, host(inputs))
    check_output(cfg, y, p.forward(), name)
    check_output(cfg, y, y_ref.float().cpu().double().numpy(), name + " vs moe_forward")
