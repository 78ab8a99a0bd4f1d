"""moe_forward_noalloc: the forward on the library's own static scratch array.

Callers that cannot allocate device memory (a plugin inside a runtime that
owns all device memory, a request path that must not call cudaMalloc) use this
entry point instead of passing a workspace.  This file is collected last so
that a run stopping at its first failure has already run every other test.
"""
import pytest
import torch

from workloads import CONFIGS, make_inputs, small

pytestmark = pytest.mark.gpu


def _cfg(seed):
    return small(CONFIGS["decode_T64"], name="noalloc", T=96, d=512, F=384, E=32, k=4, seed=seed)


def test_noalloc_entry_matches_moe_forward_on_two_calls_in_a_row():
    """Both entry points run the same bitwise-reproducible forward, one on a caller
    workspace and one on the static array, so their outputs must be identical; two
    calls in a row with different inputs also show that nothing stale from the
    previous call's scratch contents leaks into the next."""
    import mixture_experts_ffn_10_b200 as m
    stream = torch.cuda.current_stream().cuda_stream
    for seed in (2101, 2102):
        cfg = _cfg(seed)
        inputs = make_inputs(cfg, "cuda")
        ref = m.forward(cfg, inputs)          # the existing entry point, caller workspace
        y = torch.full_like(inputs["x"], float("nan"))
        shape, opts = m.shape_of(cfg), m.options_of(cfg)
        assert m.moe_workspace_size(shape, opts) <= m.moe_noalloc_workspace_bytes()
        rc = m.moe_forward_noalloc(shape, opts, m.tensors_of(inputs, y), stream)
        assert rc == m.MOE_OK, m.moe_last_error()
        assert m.moe_noalloc_debug_status(stream) == m.MOE_OK
        torch.cuda.synchronize()
        assert torch.equal(y, ref)


def test_noalloc_entry_rejects_problems_beyond_its_scratch():
    import mixture_experts_ffn_10_b200 as m
    cfg = small(CONFIGS["mixtral_bf16"], T=4096)
    shape, opts = m.shape_of(cfg), m.options_of(cfg)
    assert m.moe_workspace_size(shape, opts) > m.moe_noalloc_workspace_bytes()
    t = m.moe_tensors()
    fake = 1 << 20
    for n in ("x", "router_logits", "gate_up", "down"):
        setattr(t, n, fake)
    t.y = 2 * fake
    rc = m.moe_forward_noalloc(shape, opts, t, torch.cuda.current_stream().cuda_stream)
    assert rc == m.MOE_ERR_WORKSPACE
    assert "static array" in m.moe_last_error()
