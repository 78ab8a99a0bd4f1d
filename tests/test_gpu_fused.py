"""GPU checks of the one-launch gate_up + down GEMMs for small batches (bf16, T <= 64:
x read in place, each expert's down tiles start once its h rows are complete), and of
split-K with the last split of each tile region reducing it.

The fused launch computes what the two launches compute, with the same tiles, splits
and epilogues: the outputs must be bitwise equal with MOE_B200_FUSED_FFN=0 and =1,
and within the parity tolerance of the oracle (1e-4 of max|y| for fp32, 2e-2 bf16)."""
import pytest
import torch

from workloads import CONFIGS, make_inputs, small

from gpu_cases import parity, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _tensor_core_path(monkeypatch):
    """These cases test the tensor-core GEMMs: batches of at most 4 tokens would
    otherwise run the few-token kernel (tests/test_gpu_gemv.py)."""
    monkeypatch.setenv("MOE_B200_GEMV", "0")

DEC = small(CONFIGS["decode_T1"], name="f_decode", d=512, F=256, E=32)
CASES = {
    "T1": DEC,
    "T1_shared_gate": small(DEC, name="T1_shared_gate", Fs=192, shared_gate=True),
    "T5_unfused_bias": small(DEC, name="T5_unfused_bias", T=5, gu_layout="unfused", expert_bias=True),
    "T8_plain_gelu": small(DEC, name="T8_plain_gelu", T=8, ffn="plain", act="gelu_tanh", expert_bias=True),
    "T17_weigh_inputs": small(DEC, name="T17_weigh_inputs", T=17, weigh_inputs=True, k=4),
    "T33_abox64_interleaved": small(DEC, name="T33_abox64_interleaved", T=33, gu_layout="interleaved",
                                     act="silu", alpha=1.702, limit=7.0, expert_bias=True),
    "T64_ragged": small(DEC, name="T64_ragged", T=64, d=200, F=136, E=12, k=3, Fs=72),
    "T3_sigmoid_groups": small(CONFIGS["deepseek_bf16"], name="T3_sigmoid_groups", T=3, d=256, F=128, E=64,
                               k=8, Fs=128),
    # the router weight in front of the routing
    "T40_router": small(DEC, name="T40_router", T=40, router="weight", router_bias=True),
    "T64_router_many_experts": small(DEC, name="T64_router_many_experts", T=64, E=700, k=5, router="weight"),
}


def _both(cfg, monkeypatch):
    import mixture_experts_ffn_10_b200 as m
    inputs = make_inputs(cfg, "cuda")
    out = {}
    for flag in ("1", "0"):
        monkeypatch.setenv("MOE_B200_FUSED_FFN", flag)
        assert m.moe_forward_fused_gemms(m.shape_of(cfg), m.options_of(cfg)) == int(flag)
        y, idx, w = run_gpu(cfg, inputs)
        torch.cuda.synchronize()
        out[flag] = (y.clone(), idx.clone(), w.clone())
    return out


@pytest.mark.parametrize("name", list(CASES))
def test_fused_launch_is_bitwise_equal_to_two_launches(name, monkeypatch):
    out = _both(CASES[name], monkeypatch)
    for a, b in zip(out["1"], out["0"]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("name", list(CASES))
def test_fused_launch_matches_oracle(name):
    parity(CASES[name])


@pytest.mark.parametrize("name", ["decode_T1", "decode_T8", "decode_T64"])
def test_fused_launch_at_full_size(name, monkeypatch):
    """The decode workloads themselves (E=128, d=4096, F=1536): the fused launch, with
    gate_up split 3 ways at T=1, equals the two launches bit for bit."""
    out = _both(CONFIGS[name], monkeypatch)
    for a, b in zip(out["1"], out["0"]):
        assert torch.equal(a, b)


def test_repeated_calls_reset_the_counters():
    """The split-K and h-readiness counters are cleared by every call's sort: three
    calls in a row on one workspace give the same output."""
    import mixture_experts_ffn_10_b200 as m
    cfg = CASES["T1_shared_gate"]
    inputs = make_inputs(cfg, "cuda")
    shape, opts = m.shape_of(cfg), m.options_of(cfg)
    ws = m.Workspace(m.moe_workspace_size(shape, opts))
    ys = [m.forward(cfg, inputs, workspace=ws).clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert m.moe_debug_status(ws.ptr, torch.cuda.current_stream().cuda_stream) == 0
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])
