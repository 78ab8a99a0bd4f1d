"""GPU parity of the bf16 GEMMs with swapped operands on CTA pairs (256 weight rows
over two SMs as the MMA's M, the tile's token rows as its N, padded to 16 only).

The library picks them by itself for batches of more than 4096 routed rows (with
a fused or plain layout); MOE_B200_SWAP_GEMM=0 turns them off.  Cases span
token tiles of every height (1 .. 256 rows, the MMA's N split evenly across the
pair), ragged d and F against the 256-row weight tiles and the 64-deep K step,
both fused layouts (gate and up rows of a feature adjacent through a feature-outer
view of the stack), the plain FFN, biases, weigh-inputs and a shared expert with
its gate.  Each case is compared with the oracle and with the other kernels.
"""
import pytest
import torch

import oracle
from workloads import CONFIGS, make_inputs, small

from gpu_cases import check_output, host, parity, run_gpu

pytestmark = pytest.mark.gpu

DSK = small(CONFIGS["deepseek_bf16"], name="swap_deepseek", T=600, d=256, F=160, E=64, k=8, Fs=192)
MIX = small(CONFIGS["mixtral_bf16"], name="swap_mixtral", T=2100, d=328, F=200, E=4, k=2)

CASES = {
    "swap_deepseek": DSK,
    "swap_deepseek_shared_gate": small(DSK, name="swap_deepseek_shared_gate", shared_gate=True,
                                       shared_output=True, expert_bias=True),
    "swap_interleaved_gelu": small(DSK, name="swap_interleaved_gelu", gu_layout="interleaved",
                                   act="gelu_tanh", expert_bias=True, Fs=0, score="softmax",
                                   selection_bias_std=0.0, n_group=0, topk_group=0),
    "swap_weigh_inputs": small(DSK, name="swap_weigh_inputs", weigh_inputs=True, renormalize=False,
                               Fs=0),
    "swap_plain": small(DSK, name="swap_plain", ffn="plain", act="relu", expert_bias=True, F=328),
    "swap_large_experts": MIX,
    "swap_skewed": small(MIX, name="swap_skewed", E=32, k=2, T=2200, logits="zipf", d=256, F=256),
}


@pytest.fixture
def force_swap(monkeypatch):
    monkeypatch.setenv("MOE_B200_SWAP_GEMM", "1")


@pytest.mark.parametrize("name", list(CASES))
def test_swap_gemm_matches_oracle(name, force_swap):
    parity(CASES[name])


@pytest.mark.parametrize("name", ["swap_deepseek", "swap_large_experts"])
def test_swap_gemm_agrees_with_other_kernels_and_is_deterministic(name, monkeypatch):
    cfg = CASES[name]
    inputs = make_inputs(cfg, "cuda")
    p = oracle.Problem(cfg, host(inputs))
    ref = p.forward()
    monkeypatch.setenv("MOE_B200_SWAP_GEMM", "1")
    y1, i1, _ = run_gpu(cfg, inputs)
    y2, i2, _ = run_gpu(cfg, inputs)
    monkeypatch.setenv("MOE_B200_SWAP_GEMM", "0")
    y0, i0, _ = run_gpu(cfg, inputs)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(i1, i2), "swap kernel not deterministic"
    assert torch.equal(i0, i1)
    check_output(cfg, y1, ref, "swap")
    check_output(cfg, y0, ref, "other kernels")
