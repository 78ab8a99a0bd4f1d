"""GPU parity of the CTA-pair bf16 GEMMs (256 x 256 tiles computed by two SMs).

The library picks the pair kernels by itself for large batches (on average 512
or more routed rows per expert); MOE_B200_PAIR_GEMM=1 forces them, so that small
cases with ragged tails in every dimension (rows per expert, d against the
64-deep K step and the 256-wide N tile, F against the 128-feature gate_up tile),
both gate_up layouts, biases, a shared expert and weigh-inputs all run through
them.  Each case is compared with the oracle like the other parity tests.
"""
import pytest
import torch

import oracle
from workloads import CONFIGS, make_inputs, small

from gpu_cases import check_output, host, parity, run_gpu

pytestmark = pytest.mark.gpu

MIX = small(CONFIGS["mixtral_bf16"], name="pair_mixtral", T=700, d=328, F=200, E=4, k=2)
DSK = small(CONFIGS["deepseek_bf16"], name="pair_deepseek", T=300, d=256, F=160, E=16, k=4, Fs=192)

CASES = {
    "pair_mixtral": MIX,
    "pair_interleaved": small(MIX, name="pair_interleaved", gu_layout="interleaved", act="gelu_tanh",
                              expert_bias=True, weigh_inputs=True),
    "pair_shared_expert": small(DSK, name="pair_shared_expert", shared_gate=True, shared_output=True,
                                expert_bias=True),
    "pair_relu_beta": small(MIX, name="pair_relu_beta", act="relu", beta=0.5, T=513),
    "pair_T1": small(MIX, name="pair_T1", T=1),
    "pair_many_experts": small(MIX, name="pair_many_experts", E=64, k=8, T=200, d=256, F=256),
    "pair_skewed_top1": small(MIX, name="pair_skewed_top1", T=1024, d=512, F=256, E=2, k=1,
                              logits="zipf"),
    # the unfused gate stack and the plain (non-gated) FFN ("MoE" graph-op fc3 / fusion_size 1)
    "pair_unfused": small(DSK, name="pair_unfused", gu_layout="unfused", expert_bias=True, shared_gate=True),
    "pair_plain": small(DSK, name="pair_plain", ffn="plain", act="gelu_erf", expert_bias=True, F=328),
}


@pytest.fixture
def force_pair(monkeypatch):
    monkeypatch.setenv("MOE_B200_SWAP_GEMM", "0")
    monkeypatch.setenv("MOE_B200_PAIR_GEMM", "1")


@pytest.mark.parametrize("name", list(CASES))
def test_pair_gemm_matches_oracle(name, force_pair):
    parity(CASES[name])


def test_pair_and_single_cta_agree(monkeypatch):
    """Both GEMM variants on one problem: each within tolerance of the oracle."""
    cfg = small(MIX, name="pair_vs_single", T=900)
    inputs = make_inputs(cfg, "cuda")
    p = oracle.Problem(cfg, host(inputs))
    ref = p.forward()
    errs = {}
    monkeypatch.setenv("MOE_B200_SWAP_GEMM", "0")
    for flag in ("0", "1"):
        monkeypatch.setenv("MOE_B200_PAIR_GEMM", flag)
        y, _, _ = run_gpu(cfg, inputs)
        torch.cuda.synchronize()
        errs[flag] = check_output(cfg, y, ref, f"MOE_B200_PAIR_GEMM={flag}")
    assert max(errs.values()) < 2e-2


def test_pair_gemm_deterministic(force_pair):
    cfg = small(MIX, name="pair_determinism", T=1500)
    inputs = make_inputs(cfg, "cuda")
    y1, i1, _ = run_gpu(cfg, inputs)
    y2, i2, _ = run_gpu(cfg, inputs)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
