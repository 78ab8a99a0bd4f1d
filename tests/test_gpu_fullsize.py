"""Parity at the full workload sizes the benchmark times (same entry point and launch).

Every token's routing is compared bit-exactly with the oracle.  Outputs are
compared element by element on a sample of tokens that the oracle computes one
by one: for every expert that receives rows, the tokens of its first and last
row and of the rows on both sides of every 128-row boundary inside its segment
(the GEMM tile edges of both the 128- and the 256-row tiles), up to a budget,
plus the first and last token of the batch; batches of at most 256 tokens are
compared on every token.  The forward is run twice to check bitwise
determinism at full size.  Weights of experts the sampled tokens do not use are
never copied to the host (the host arrays are lazily zero-filled).
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, make_inputs

from gpu_cases import TOL, W_RTOL, run_gpu

pytestmark = pytest.mark.gpu

FULL = ["tiny_fp32", "mixtral_bf16", "gptoss_mxfp4", "deepseek_bf16", "decode_T1", "decode_T8",
        "decode_T64", "decode_T256"]
MAX_SAMPLE = 160   # tokens the oracle recomputes per workload (about 10-15 s on 16 host cores)
ALL_TOKENS_UP_TO = 256


def _np(t):
    t = t.detach()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    return t


def boundary_sample(idx, E, seed, budget=MAX_SAMPLE, tile=128):
    """Tokens whose rows sit at the edges of each expert's segment and of its
    row tiles (rows are token-ascending inside an expert's segment)."""
    T = idx.shape[0]
    if T <= ALL_TOKENS_UP_TO:
        return list(range(T))
    per_expert = [[] for _ in range(E)]
    for t, row in enumerate(idx.tolist()):
        for e in row:
            per_expert[e].append(t)
    # one list of edge tokens per expert, nearest edges first
    edges = []
    for toks in per_expert:
        n = len(toks)
        if n == 0:
            continue
        pos = [0, n - 1]
        for b in range(tile, n, tile):
            pos += [b - 1, b]
        edges.append([toks[i] for i in dict.fromkeys(pos)])
    rng = np.random.default_rng(seed)
    rng.shuffle(edges)
    chosen = {0, T - 1}
    depth = 0
    # round robin over the experts: every expert's first edge, then every second, ...
    while len(chosen) < budget and any(depth < len(e) for e in edges):
        for e in edges:
            if depth < len(e):
                chosen.add(e[depth])
                if len(chosen) >= budget:
                    break
        depth += 1
    return sorted(chosen)


def _host_sparse(inputs, experts):
    """Host copies: small tensors whole, expert stacks only for `experts` (rest lazily zero)."""
    out = {}
    for k, v in inputs.items():
        if v is None:
            out[k] = None
            continue
        a = _np(v)
        if k in ("gate_up", "down", "gate_up_scales", "down_scales"):
            dt = {torch.int16: np.uint16, torch.uint8: np.uint8, torch.float32: np.float32}[a.dtype]
            h = np.zeros(tuple(a.shape), dtype=dt)  # calloc: untouched experts cost no memory
            for e in experts:
                h[e] = a[e].cpu().numpy().view(dt)
            out[k] = h
        else:
            h = a.cpu().numpy()
            out[k] = h.view(np.uint16) if a.dtype == torch.int16 else h
    return out


@pytest.mark.parametrize("name", FULL)
def test_full_size_parity(name):
    _full_size(name)


@pytest.mark.parametrize("pair", ["0", "1"], ids=["single_cta", "token_tile_pair"])
def test_full_size_mixtral_token_tile_gemms(monkeypatch, pair):
    """The large-batch workload again on the token-tile GEMMs (the library picks the
    swapped-operand CTA-pair GEMMs for it by default): one CTA per 128-row tile, and
    CTA pairs per 256-row tile."""
    monkeypatch.setenv("MOE_B200_SWAP_GEMM", "0")
    monkeypatch.setenv("MOE_B200_PAIR_GEMM", pair)
    _full_size("mixtral_bf16")


def _full_size(name):
    cfg = CONFIGS[name]
    torch.manual_seed(0)
    inputs = make_inputs(cfg, "cuda")
    y, idx, w = run_gpu(cfg, inputs)
    y2, idx2, _ = run_gpu(cfg, inputs)
    torch.cuda.synchronize()
    assert torch.equal(y, y2) and torch.equal(idx, idx2), "not bitwise reproducible at full size"

    # routing of every token
    idx_h, w_h = idx.cpu().numpy(), w.cpu().numpy()
    routing_only = {k: inputs[k] for k in ("logits", "router_bias", "selection_bias")}
    pr = oracle.Problem(cfg, {k: (None if v is None else v.cpu()) for k, v in routing_only.items()})
    sample = boundary_sample(idx.cpu().numpy(), cfg.E, cfg.seed)
    for t in range(cfg.T):
        ri, rw, _, _ = pr.route(t)
        assert np.array_equal(idx_h[t], ri), f"token {t}: {idx_h[t]} vs {ri}"
        assert np.all(np.abs(w_h[t] - rw) <= W_RTOL * np.abs(rw) + 1e-30)

    # outputs of the sampled tokens
    experts = sorted({int(e) for t in sample for e in idx_h[t]})
    p = oracle.Problem(cfg, _host_sparse(inputs, experts))
    ref = p.forward(np.array(sample, dtype=np.int64))
    got = y[sample].float().cpu().double().numpy()
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert np.isfinite(got).all()
    assert err <= TOL[cfg.act_dtype] * scale, f"{name}: max err {err:.3e} > {TOL[cfg.act_dtype] * scale:.3e}"
