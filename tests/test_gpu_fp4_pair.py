"""GPU parity of the CTA-pair MXFP4 GEMMs (256 decoded weight rows over two SMs).

The library picks them by itself when the routed rows average at least 128 per
expert; MOE_B200_PAIR_FP4=1 forces them, so that small cases run through them
too: token tiles of every height (1 .. 256 rows, the MMA's N split evenly across
the pair), ragged d and F against the 256-row weight tiles, both fused layouts,
the unfused gate stack, the plain FFN, biases and weigh-inputs.  Each case is
compared with the oracle, with the single-CTA MXFP4 kernels (same arithmetic, to
within one bf16 rounding of the stored activations), and against itself for
determinism.
"""
import pytest
import torch

from workloads import CONFIGS, make_inputs, small

from gpu_cases import parity, run_gpu

pytestmark = pytest.mark.gpu

FP4 = small(CONFIGS["gptoss_mxfp4"], name="fp4p", T=300, d=320, F=352, E=6, k=3)

CASES = {
    "fp4p_base": FP4,
    "fp4p_concat": small(FP4, name="fp4p_concat", gu_layout="concat", limit=0.0, alpha=1.0),
    "fp4p_three_tiles": small(FP4, name="fp4p_three_tiles", T=600, E=2, k=2, d=256, F=256),
    "fp4p_T1": small(FP4, name="fp4p_T1", T=1, E=32, k=4),
    "fp4p_T7": small(FP4, name="fp4p_T7", T=7),
    "fp4p_unfused": small(FP4, name="fp4p_unfused", gu_layout="unfused"),
    "fp4p_plain": small(FP4, name="fp4p_plain", ffn="plain", act="gelu_tanh"),
    "fp4p_weigh_inputs": small(FP4, name="fp4p_weigh_inputs", weigh_inputs=True, renormalize=False),
    "fp4p_wide": small(FP4, name="fp4p_wide", d=1024, F=544, T=513, E=4, k=2),
    "fp4p_shared_expert": small(FP4, name="fp4p_shared_expert", Fs=320, shared_gate=True, shared_output=True),
}


@pytest.fixture
def force_pair_fp4(monkeypatch):
    monkeypatch.setenv("MOE_B200_PAIR_FP4", "1")


@pytest.mark.parametrize("name", list(CASES))
def test_pair_fp4_matches_oracle(name, force_pair_fp4):
    parity(CASES[name])


@pytest.mark.parametrize("name", ["fp4p_base", "fp4p_three_tiles", "fp4p_plain", "fp4p_unfused"])
def test_pair_fp4_agrees_with_single_cta_kernel(name, monkeypatch):
    cfg = CASES[name]
    inputs = make_inputs(cfg, "cuda")
    monkeypatch.setenv("MOE_B200_PAIR_FP4", "0")
    y1, i1, _ = run_gpu(cfg, inputs)
    monkeypatch.setenv("MOE_B200_PAIR_FP4", "1")
    y2, i2, _ = run_gpu(cfg, inputs)
    y3, _, _ = run_gpu(cfg, inputs)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2)
    assert torch.equal(y2, y3), "pair kernel not deterministic"
    a, b = y2.float(), y1.float()
    assert (a - b).abs().max().item() <= 1e-2 * b.abs().max().item(), "pair and single-CTA kernels differ"
