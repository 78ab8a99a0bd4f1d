"""The expert-parallel exchange on CPU: 2 and 4 gloo ranks, uneven token counts.

The device steps (routing, permute, expert FFNs, combine) are replaced by a stand-in
built on the oracle (test infrastructure: the oracle's routing and its per-expert FFN,
numpy for the row order); what is under test is the module's exchange -- the split
sizes, the all-to-alls of rows, experts and weights, the return of the outputs and
their placement for the combine.  Each rank's y must match the oracle's forward of
its tokens with all experts on one device (to the fp32 rounding of the routing
weights that travel with the rows)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _host(t):
    return None if t is None else t.detach().cpu()


class OracleOps:
    """The device steps of ExpertParallelMoE restated on the host with the oracle."""

    def __init__(self, local_cfg_base, local_tensors):
        self.local_cfg_base = local_cfg_base
        self.local_tensors = local_tensors

    def route(self, cfg, inputs):
        import oracle
        p = oracle.Problem(cfg, {k: _host(v) for k, v in inputs.items()})
        idx, w = p.route_all()
        return torch.from_numpy(idx), torch.from_numpy(w.astype(np.float32))

    def permute(self, cfg, idx, w, x, experts_per_rank):
        flat = idx.reshape(-1).numpy()
        order = np.argsort(flat, kind="stable")  # expert order, slot order within an expert
        pos = np.empty_like(order)
        pos[order] = np.arange(order.size)
        e = flat[order]
        row_expert = e % experts_per_rank if experts_per_rank > 0 else e
        return (x[torch.from_numpy(order // cfg.k)], torch.from_numpy(row_expert.astype(np.int32)),
                w.reshape(-1)[torch.from_numpy(order)], torch.from_numpy(np.bincount(flat, minlength=cfg.E)),
                torch.from_numpy(pos.reshape(cfg.T, cfg.k).astype(np.int32)))

    def experts_forward(self, cfg_local, rows, row_expert, row_w, weights):
        import oracle
        p = oracle.Problem(cfg_local, {k: _host(v) for k, v in weights.items()
                                       if k not in ("router_bias", "selection_bias")})
        xs = rows.double().numpy()
        out = np.zeros_like(xs)
        for r in range(xs.shape[0]):
            e, wr = int(row_expert[r]), float(row_w[r])
            out[r] = p.expert(e, wr * xs[r]) if cfg_local.weigh_inputs else wr * p.expert(e, xs[r])
        return torch.from_numpy(out)

    def combine(self, cfg, pos, Y, shared_output=None):
        y = Y[pos.long()].sum(dim=1)
        return y if shared_output is None else y + shared_output.double()


def _rank_main(rank, world, port, cfg, counts, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    from mixture_experts_ffn_10_b200.ep import ExpertParallelMoE
    from workloads import make_inputs, small
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        inputs = make_inputs(cfg, "cpu")  # every rank builds the same global problem
        t0 = sum(counts[:rank])
        T = counts[rank]
        El = cfg.E // world
        local = {k: (v[rank * El:(rank + 1) * El] if v is not None else None)
                 for k, v in inputs.items() if k in ("gate_up", "gate_up_bias", "down", "down_bias", "gate",
                                                     "gate_bias")}
        local["router_bias"] = inputs.get("router_bias")
        local["selection_bias"] = inputs.get("selection_bias")
        local["router_weight"] = inputs.get("router_weight")
        mine = small(cfg, T=T)
        layer = ExpertParallelMoE(mine, local, ops=OracleOps(mine, local))
        logits = inputs["logits"][t0:t0 + T] if inputs.get("logits") is not None else None
        y = layer.forward(inputs["x"][t0:t0 + T], logits)
        out[rank] = y.numpy()
    finally:
        dist.destroy_process_group()


VARIANTS = {
    "concat": dict(gu_layout="concat", expert_bias=True),
    "interleaved": dict(gu_layout="interleaved", expert_bias=True),
    "unfused_weigh_inputs": dict(gu_layout="unfused", expert_bias=True, weigh_inputs=True),
    "plain_relu": dict(ffn="plain", act="relu"),
    "sigmoid_groups_bias": dict(score="sigmoid", n_group=4, topk_group=2, renormalize=True, routed_scale=2.5,
                                selection_bias_std=0.1, router_bias=True),
    "router_weight": dict(router="weight", router_bias=True),
}


@pytest.mark.parametrize("world,counts,variant", [
    (2, [7, 5], "concat"), (4, [3, 0, 6, 2], "interleaved"), (2, [4, 9], "unfused_weigh_inputs"),
    (2, [6, 6], "plain_relu"), (4, [5, 2, 3, 4], "sigmoid_groups_bias"), (2, [5, 8], "router_weight")])
def test_expert_parallel_exchange_matches_one_device(world, counts, variant):
    sys.path.insert(0, ROOT)
    import oracle
    from workloads import CONFIGS, make_inputs, small
    cfg = small(CONFIGS["decode_T1"], name="ep_cpu", T=sum(counts), d=64, F=32, E=8, k=3,
                act_dtype="f32", w_dtype="f32", logit_dtype="f32", **VARIANTS[variant])
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), cfg, counts, out), nprocs=world, join=True)
        res = dict(out)
    inputs = make_inputs(cfg, "cpu")
    ref = oracle.Problem(cfg, {k: _host(v) for k, v in inputs.items()}).forward()
    t0 = 0
    for r in range(world):
        got = res[r]
        assert got.shape == (counts[r], cfg.d)
        np.testing.assert_allclose(got, ref[t0:t0 + counts[r]], rtol=1e-6, atol=1e-6)  # fp32 routing weights
        t0 += counts[r]
