"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare (routing bit-exact, outputs within tolerance)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from workloads import make_inputs

# Output tolerance: max|y_gpu - y_oracle| <= TOL * max|y_oracle| (fp32 accumulation
# everywhere; bf16 inputs/outputs and bf16 intermediate activations).
TOL = {"f32": 1e-4, "bf16": 2e-2}
W_RTOL = 1e-6   # routing weights (double on both sides, rounded once to fp32)


def moe_lib():
    import mixture_experts_ffn_10_b200 as m
    return m


def host(inputs: dict) -> dict:
    return {k: (None if v is None else v.detach().cpu()) for k, v in inputs.items()}


def run_gpu(cfg, inputs, with_route=True):
    m = moe_lib()
    shape, opts = m.shape_of(cfg), m.options_of(cfg)
    ws = m.Workspace(m.moe_workspace_size(shape, opts))
    idx = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda") if with_route else None
    w = torch.full((cfg.T, cfg.k), -7.0, dtype=torch.float32, device="cuda") if with_route else None
    y = m.forward(cfg, inputs, workspace=ws, topk_idx=idx, topk_w=w)
    status = m.moe_debug_status(ws.ptr, torch.cuda.current_stream().cuda_stream)
    assert status == 0, f"device status {m.STATUS_NAMES.get(status, status)}"
    return y, idx, w


def near_tie_report(keys, a, b):
    """Describe the key gaps of experts that differ between two selections."""
    diff = sorted(set(a.tolist()) ^ set(b.tolist()))
    return ", ".join(f"e{e}: key={keys[e]!r}" for e in diff)


def check_routing(p, idx, w, tokens=None):
    idx = idx.cpu().numpy()
    w = w.cpu().numpy()
    tokens = range(idx.shape[0]) if tokens is None else tokens
    for t in tokens:
        ri, rw, keys, _ = p.route(int(t))
        assert np.array_equal(idx[t], ri), (
            f"token {t}: gpu {idx[t].tolist()} oracle {ri.tolist()} ({near_tie_report(keys, idx[t], ri)})")
        assert np.all(np.abs(w[t] - rw) <= W_RTOL * np.abs(rw) + 1e-30), (t, w[t], rw)


def check_output(cfg, y_gpu, y_ref, what=""):
    y = y_gpu.float().cpu().double().numpy()
    scale = np.abs(y_ref).max()
    err = np.abs(y - y_ref).max()
    assert np.isfinite(y).all(), f"{what}: non-finite output"
    assert err <= TOL[cfg.act_dtype] * scale, f"{what}: max err {err:.3e} vs tol {TOL[cfg.act_dtype] * scale:.3e}"
    return err / scale


def parity(cfg, override=None):
    """Full forward parity on every token; returns the relative error."""
    inputs = make_inputs(cfg, "cuda")
    if override:
        inputs.update({k: (v.cuda() if v is not None else None) for k, v in override.items()})
    y, idx, w = run_gpu(cfg, inputs)
    torch.cuda.synchronize()
    p = oracle.Problem(cfg, host(inputs))
    check_routing(p, idx, w)
    return check_output(cfg, y, p.forward(), cfg.name)
