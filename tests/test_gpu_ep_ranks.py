"""The expert-parallel layer with its real device steps on two ranks: two processes on
one GPU, each running the library's kernels on its own tokens and its half of the
experts, exchanging rows through host memory over gloo (the kernels of the two ranks
never wait on one another; only the host-side collectives synchronise them).  Each
rank's y must match the oracle's forward of its tokens and moe_forward with all the
experts on one rank."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, cfg, counts, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import mixture_experts_ffn_10_b200 as m
    from mixture_experts_ffn_10_b200.ep import ExpertParallelMoE
    from workloads import make_inputs, small
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        inputs = make_inputs(cfg, "cuda")  # every rank builds the same global problem
        t0, T = sum(counts[:rank]), counts[rank]
        El = cfg.E // world
        local = {k: (v[rank * El:(rank + 1) * El].contiguous() if v is not None else None)
                 for k, v in inputs.items() if k in ("gate_up", "gate_up_scales", "gate_up_bias", "down",
                                                     "down_scales", "down_bias", "gate", "gate_bias")}
        local["router_bias"], local["selection_bias"] = inputs.get("router_bias"), inputs.get("selection_bias")
        mine = small(cfg, T=T)
        x, logits = inputs["x"][t0:t0 + T].contiguous(), inputs["logits"][t0:t0 + T].contiguous()
        y = ExpertParallelMoE(mine, local).forward(x, logits)
        mine_inputs = dict(inputs, x=x, logits=logits)
        y_one = m.forward(mine, mine_inputs)
        torch.cuda.synchronize()
        out[rank] = (y.float().cpu().numpy(), y_one.float().cpu().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", ["bf16", "mxfp4"])
def test_two_ranks_on_the_library_kernels(name):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from gpu_cases import TOL, host
    from workloads import CONFIGS, make_inputs, small
    if name == "bf16":
        cfg = small(CONFIGS["decode_T1"], name="ep_ranks", T=90, d=256, F=128, E=16, k=4, expert_bias=True)
    else:
        cfg = small(CONFIGS["gptoss_mxfp4"], name="ep_ranks_fp4", T=90, d=320, F=352, E=8, k=4)
    counts = [53, 37]
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(2, _free_port(), cfg, counts, out), nprocs=2, join=True)
        res = dict(out)
    inputs = make_inputs(cfg, "cuda")  # the ranks' inputs (the device generator's stream)
    ref = oracle.Problem(cfg, host(inputs)).forward()
    t0 = 0
    for r in range(2):
        y, y_one = res[r]
        want = ref[t0:t0 + counts[r]]
        scale = np.abs(want).max()
        errs = (np.abs(y - want).max(), np.abs(y - y_one).max(), np.abs(y_one - want).max())
        assert max(errs) <= TOL[cfg.act_dtype] * scale, (r, errs, scale)
        t0 += counts[r]
