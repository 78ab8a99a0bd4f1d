"""GPU checks of the few-token forward (bf16 weights, T <= 4): routing, gate_up,
down and the combine in one launch of the CUDA-core kernel.

Against the oracle on every token (routing bit-exact, outputs within 2e-2 of max|y|),
over every layout, activation and option the kernel serves, at small and at the
decode workloads' full sizes; bitwise repeatable from run to run; and within the same
tolerance of the multi-launch tensor-core path (MOE_B200_GEMV=0)."""
import pytest
import torch

from workloads import CONFIGS, make_inputs, small

from gpu_cases import check_output, parity, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _few_token_kernel(monkeypatch):
    """The kernel is opt-in: MOE_B200_GEMV=4 turns it on for batches of up to 4 tokens."""
    monkeypatch.setenv("MOE_B200_GEMV", "4")

DEC = small(CONFIGS["decode_T1"], name="g_decode", d=512, F=256, E=32)
CASES = {
    "T1": DEC,
    "T1_k1": small(DEC, name="T1_k1", E=8, k=1),
    "T1_shared_gate": small(DEC, name="T1_shared_gate", Fs=192, shared_gate=True),
    "T2_unfused_bias": small(DEC, name="T2_unfused_bias", T=2, gu_layout="unfused", expert_bias=True),
    "T3_plain_gelu": small(DEC, name="T3_plain_gelu", T=3, ffn="plain", act="gelu_tanh", expert_bias=True),
    "T4_weigh_inputs": small(DEC, name="T4_weigh_inputs", T=4, weigh_inputs=True, k=4),
    "T2_interleaved_clamp": small(DEC, name="T2_interleaved_clamp", T=2, gu_layout="interleaved",
                                  act="silu", alpha=1.702, limit=7.0, expert_bias=True),
    # d = 192: a last K stage of 192 of 256 (the rest of the tile zero-filled by the
    # TMA); Fs = 128 beside F = 64: down stages of the routed experts stop early
    "T4_ragged_shared": small(DEC, name="T4_ragged_shared", T=4, d=192, F=64, E=12, k=3, Fs=128),
    "T4_plain_shared_output": small(DEC, name="T4_plain_shared_output", T=4, ffn="plain", act="relu", Fs=64,
                                    shared_output=True),
    "T3_sigmoid_groups": small(CONFIGS["deepseek_bf16"], name="T3_sigmoid_groups", T=3, d=256, F=128, E=64,
                               k=8, Fs=128),
    "T4_k32": small(DEC, name="T4_k32", T=4, E=64, k=32, F=64),
    "T2_router": small(DEC, name="T2_router", T=2, router="weight", router_bias=True),
    "T1_router_shared_gate": small(DEC, name="T1_router_shared_gate", router="weight", Fs=64, shared_gate=True),
}


def _kernel_is_gemv(cfg):
    import mixture_experts_ffn_10_b200 as m
    return m.moe_forward_fused_gemms(m.shape_of(cfg), m.options_of(cfg)) == 2


@pytest.mark.parametrize("name", list(CASES))
def test_gemv_matches_oracle(name):
    cfg = CASES[name]
    assert _kernel_is_gemv(cfg)
    parity(cfg)


@pytest.mark.parametrize("T", [1, 2, 4])
def test_gemv_at_decode_size(T):
    """The decode workload's layer (d=4096, F=1536, E=128, k=8) at T = 1, 2, 4."""
    cfg = CONFIGS["decode_T1"] if T == 1 else small(CONFIGS["decode_T1"], name=f"decode_T{T}", T=T)
    assert _kernel_is_gemv(cfg)
    parity(cfg)


@pytest.mark.parametrize("name", ["T1", "T4_ragged_shared", "T2_router"])
def test_gemv_is_repeatable_and_resets_its_counter(name):
    """Three calls on one workspace: the CTA counter is cleared by each call, and the
    fixed-order sums give the same bits every time."""
    import mixture_experts_ffn_10_b200 as m
    cfg = CASES[name]
    inputs = make_inputs(cfg, "cuda")
    shape, opts = m.shape_of(cfg), m.options_of(cfg)
    ws = m.Workspace(m.moe_workspace_size(shape, opts))
    ys = [m.forward(cfg, inputs, workspace=ws).clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert m.moe_debug_status(ws.ptr, torch.cuda.current_stream().cuda_stream) == 0
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


@pytest.mark.parametrize("name", ["T1_shared_gate", "T3_plain_gelu", "T4_weigh_inputs"])
def test_gemv_agrees_with_the_tensor_core_path(name, monkeypatch):
    """Same routing bit for bit; outputs within the parity tolerance of each other
    (the dot products sum in another order)."""
    cfg = CASES[name]
    inputs = make_inputs(cfg, "cuda")
    y1, i1, w1 = run_gpu(cfg, inputs)
    monkeypatch.setenv("MOE_B200_GEMV", "0")
    assert not _kernel_is_gemv(cfg)
    y0, i0, w0 = run_gpu(cfg, inputs)
    torch.cuda.synchronize()
    assert torch.equal(i1, i0) and torch.equal(w1, w0)
    check_output(cfg, y1, y0.float().cpu().double().numpy(), name)


def test_shapes_outside_the_kernel_fall_back():
    """d, F or Fs not in whole 64-element blocks: the multi-launch path, still exact."""
    cfg = small(DEC, name="T2_ragged_fallback", T=2, d=200, F=136, E=12, k=3, Fs=72)
    assert not _kernel_is_gemv(cfg)
    parity(cfg)
