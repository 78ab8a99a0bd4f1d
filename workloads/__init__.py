"""Seeded synthetic MoE workloads: shapes, options and input tensors.

This module is shared by the tests and the benchmark to feed the same bits to
the CUDA library and to the CPU oracle.  It draws random numbers and encodes
them into the input formats (bf16, fp32, and the MXFP4 weight payload); it
holds none of the forward pass's arithmetic.

Recipe (every tensor has its own generator, seeded ``seed * 1000 + slot``):
  x ~ N(0, 1); router logits ~ N(0, 1) (optionally minus s * ln(rank), a Zipf
  popularity prior with rank a seeded permutation of 1..E); expert weights and
  biases ~ N(0, 0.02); selection bias ~ N(0, std).  Samples are drawn in fp32
  and rounded (round-to-nearest-even) to the stored dtype.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import torch

__all__ = ["MoeConfig", "CONFIGS", "make_inputs", "quantize_mxfp4", "flops", "algorithmic_bytes",
           "small"]


@dataclass(frozen=True)
class MoeConfig:
    name: str
    T: int
    d: int
    F: int
    E: int
    k: int
    Fs: int = 0                     # shared expert dff; 0 = none
    act_dtype: str = "bf16"         # x, y, biases, shared weights
    w_dtype: str = "bf16"           # routed expert stacks: f32 | bf16 | mxfp4
    logit_dtype: str = "bf16"       # router logits and router bias
    score: str = "softmax"          # softmax | sigmoid
    renormalize: bool = True
    routed_scale: float = 1.0
    n_group: int = 0
    topk_group: int = 0
    weigh_inputs: bool = False
    act: str = "silu"               # silu | gelu_erf | gelu_tanh | relu | identity
    alpha: float = 1.0
    beta: float = 0.0
    limit: float = 0.0
    gu_layout: str = "concat"       # concat (gate rows first) | interleaved (even rows gate) | unfused
    ffn: str = "gated"              # gated: act(gate) * (up + beta) | plain: act(fc1) alone
    router: str = "logits"          # logits: caller's router logits | weight: logits = x Wr in the layer
    shared_gate: bool = False
    router_bias: bool = False
    expert_bias: bool = False
    selection_bias_std: float = 0.0  # 0 = no selection bias
    logits: str = "normal"          # normal | zipf
    zipf_s: float = 1.1
    shared_output: bool = False
    seed: int = 1000
    extra: dict = field(default_factory=dict, compare=False, hash=False)


CONFIGS = {
    "tiny_fp32": MoeConfig("tiny_fp32", T=64, d=128, F=256, E=8, k=2, act_dtype="f32",
                           w_dtype="f32", logit_dtype="f32", seed=1001),
    "mixtral_bf16": MoeConfig("mixtral_bf16", T=4096, d=4096, F=14336, E=8, k=2, seed=1002),
    "gptoss_mxfp4": MoeConfig("gptoss_mxfp4", T=2048, d=2880, F=2880, E=32, k=4, w_dtype="mxfp4",
                              gu_layout="interleaved", alpha=1.702, limit=7.0, router_bias=True,
                              expert_bias=True, seed=1003),
    "deepseek_bf16": MoeConfig("deepseek_bf16", T=8192, d=7168, F=2048, E=256, k=8, Fs=2048,
                               score="sigmoid", selection_bias_std=0.1, n_group=8, topk_group=4,
                               routed_scale=2.5, seed=1004),
}
for _T in (1, 8, 64, 256):
    CONFIGS[f"decode_T{_T}"] = MoeConfig(f"decode_T{_T}", T=_T, d=4096, F=1536, E=128, k=8,
                                         logits="zipf", seed=1005)


def small(cfg: MoeConfig, **kw) -> MoeConfig:
    """A copy of ``cfg`` with some fields replaced (shrunken test cases)."""
    return dataclasses.replace(cfg, **kw)


_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _gen(cfg: MoeConfig, slot: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed * 1000 + slot)
    return g


def _normal(shape, std, dtype, g, device):
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)


# e2m1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}: the points halfway between neighbours
_E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def quantize_mxfp4(w: torch.Tensor):
    """Encode fp32 weights [..., K] (K % 32 == 0) as MXFP4: (codes [..., K/2] u8, scales [..., K/32] u8).

    Encoding (OCP Microscaling v1.0 element and scale formats): per block of 32
    along K the e8m0 scale is s = floor(log2(amax)) - 2 + 127 (127 for an
    all-zero block), and each element is rounded to the nearest e2m1 value of
    x / 2^(s-127), ties to the even mantissa, saturating at +-6.  Two codes per
    byte, the even element in the low nibble.
    """
    *lead, K = w.shape
    assert K % 32 == 0
    b = w.float().reshape(*lead, K // 32, 32)
    amax = b.abs().amax(-1)
    _, ex = torch.frexp(amax)                 # amax = m * 2^ex, m in [0.5, 1)
    s = torch.where(amax > 0, ex - 1 - 2 + 127, torch.full_like(ex, 127)).clamp(0, 254)
    scaled = torch.ldexp(b, (127 - s).unsqueeze(-1).to(torch.float32))
    a = scaled.abs()
    mids = torch.tensor(_E2M1_MIDPOINTS, device=w.device, dtype=torch.float32)
    code = torch.bucketize(a, mids)           # number of midpoints strictly below a
    on_mid = (code < 7) & (a == mids[code.clamp(max=6)]) & (code % 2 == 1)
    code = code + on_mid.to(code.dtype)       # a tie goes to the even (mantissa 0) neighbour
    code = code | ((scaled < 0).to(code.dtype) << 3)
    code = code.to(torch.uint8).reshape(*lead, K)
    packed = code[..., 0::2] | (code[..., 1::2] << 4)
    return packed.contiguous(), s.to(torch.uint8).reshape(*lead, K // 32).contiguous()


def _weights(cfg, slot, e_count, rows, K, device):
    """Expert stack [e_count, rows, K] ~ N(0, 0.02), drawn expert by expert."""
    g = _gen(cfg, slot, device)
    if cfg.w_dtype == "mxfp4":
        q = torch.empty((e_count, rows, K // 2), dtype=torch.uint8, device=device)
        s = torch.empty((e_count, rows, K // 32), dtype=torch.uint8, device=device)
        for e in range(e_count):
            q[e], s[e] = quantize_mxfp4(_normal((rows, K), 0.02, torch.float32, g, device))
        return q, s
    dt = _TORCH_DTYPE[cfg.w_dtype]
    w = torch.empty((e_count, rows, K), dtype=dt, device=device)
    for e in range(e_count):
        w[e] = _normal((rows, K), 0.02, dt, g, device)
    return w, None


def make_inputs(cfg: MoeConfig, device="cpu", with_weights: bool = True) -> dict:
    """All input tensors of one forward, on ``device``.

    Keys (absent = None): x [T,d], logits [T,E], router_bias [E] (logit dtype),
    selection_bias [E] f32, gate_up [E,2F,d] (or MXFP4 codes [E,2F,d/2] with
    gate_up_scales [E,2F,d/32]), gate_up_bias [E,2F], down [E,d,F] (or codes
    [E,d,F/2] with down_scales [E,d,F/32]), down_bias [E,d], shared_gate_up
    [2Fs,d], shared_down [d,Fs], shared_gate_vec [d], shared_output [T,d].
    Unfused layout: gate [E,F,d] (+ gate_scales, gate_bias [E,F]) and gate_up holds
    the up rows [E,F,d] (bias [E,F]).  Plain FFN: gate_up is fc1 [E,F,d] (bias
    [E,F]) and the shared stack [Fs,d].  Router weight: router_weight [d,E] (act
    dtype) and logits None.
    """
    T, d, F, E = cfg.T, cfg.d, cfg.F, cfg.E
    adt = _TORCH_DTYPE[cfg.act_dtype]
    ldt = _TORCH_DTYPE[cfg.logit_dtype]
    out = dict.fromkeys(["x", "logits", "router_bias", "selection_bias", "gate_up",
                         "gate_up_scales", "gate_up_bias", "down", "down_scales", "down_bias",
                         "shared_gate_up", "shared_down", "shared_gate_vec", "shared_output",
                         "gate", "gate_scales", "gate_bias", "router_weight"])
    out["x"] = _normal((T, d), 1.0, adt, _gen(cfg, 0, device), device)
    if cfg.router == "weight":
        out["router_weight"] = _normal((d, E), 0.02, adt, _gen(cfg, 13, device), device)
    else:
        logits = torch.randn((T, E), generator=_gen(cfg, 1, device), device=device)
        if cfg.logits == "zipf":
            g = _gen(cfg, 2, device)
            rank = torch.randperm(E, generator=g, device=device).to(torch.float32) + 1.0
            logits = logits - cfg.zipf_s * torch.log(rank)
        out["logits"] = logits.to(ldt)
    if cfg.router_bias:
        out["router_bias"] = _normal((E,), 0.02, ldt, _gen(cfg, 3, device), device)
    if cfg.selection_bias_std > 0:
        out["selection_bias"] = _normal((E,), cfg.selection_bias_std, torch.float32,
                                        _gen(cfg, 4, device), device)
    separate = cfg.gu_layout == "unfused" or cfg.ffn == "plain"  # gate_up holds F rows per expert
    fc1_rows = F if separate else 2 * F
    if with_weights:
        out["gate_up"], out["gate_up_scales"] = _weights(cfg, 5, E, fc1_rows, d, device)
        out["down"], out["down_scales"] = _weights(cfg, 6, E, d, F, device)
        if cfg.gu_layout == "unfused" and cfg.ffn == "gated":
            out["gate"], out["gate_scales"] = _weights(cfg, 14, E, F, d, device)
    if cfg.expert_bias:
        out["gate_up_bias"] = _normal((E, fc1_rows), 0.02, adt, _gen(cfg, 7, device), device)
        out["down_bias"] = _normal((E, d), 0.02, adt, _gen(cfg, 8, device), device)
        if cfg.gu_layout == "unfused" and cfg.ffn == "gated":
            out["gate_bias"] = _normal((E, F), 0.02, adt, _gen(cfg, 15, device), device)
    if cfg.Fs > 0 and with_weights:
        sh_rows = cfg.Fs if cfg.ffn == "plain" else 2 * cfg.Fs
        out["shared_gate_up"] = _normal((sh_rows, d), 0.02, adt, _gen(cfg, 9, device), device)
        out["shared_down"] = _normal((d, cfg.Fs), 0.02, adt, _gen(cfg, 10, device), device)
    if cfg.shared_gate:
        out["shared_gate_vec"] = _normal((d,), 0.02, adt, _gen(cfg, 11, device), device)
    if cfg.shared_output:
        out["shared_output"] = _normal((T, d), 1.0, adt, _gen(cfg, 12, device), device)
    return out


def _mats(cfg: MoeConfig) -> int:
    """Weight matrices per expert: gate, up and down (gated) or fc1 and down (plain)."""
    return 2 if cfg.ffn == "plain" else 3


def flops(cfg: MoeConfig) -> float:
    """Algorithmic FLOPs of one forward: 2*R*m*d*F routed + 2*T*m*d*Fs shared (m = 3
    matrices per gated expert, 2 per plain one), + 2*T*d*E for a router weight."""
    m = _mats(cfg)
    f = 2.0 * cfg.T * cfg.k * m * cfg.d * cfg.F + 2.0 * cfg.T * m * cfg.d * cfg.Fs
    if cfg.router == "weight":
        f += 2.0 * cfg.T * cfg.d * cfg.E
    return f


def weight_bytes_per_expert(cfg: MoeConfig) -> float:
    n = _mats(cfg) * cfg.d * cfg.F
    if cfg.w_dtype == "mxfp4":
        b = n / 2 + n / 32
    else:
        b = n * (4 if cfg.w_dtype == "f32" else 2)
    if cfg.expert_bias:
        b += ((_mats(cfg) - 1) * cfg.F + cfg.d) * (4 if cfg.act_dtype == "f32" else 2)
    return b


def algorithmic_bytes(cfg: MoeConfig, distinct_experts: int) -> float:
    """Bytes a forward must move: touched experts' weights (+biases, scales), shared
    weights, x, the router logits (or the router weight) and y."""
    ab = 4 if cfg.act_dtype == "f32" else 2
    lb = 4 if cfg.logit_dtype == "f32" else 2
    b = distinct_experts * weight_bytes_per_expert(cfg)
    b += _mats(cfg) * cfg.d * cfg.Fs * ab
    b += cfg.T * cfg.d * ab * 2
    b += cfg.d * cfg.E * ab if cfg.router == "weight" else cfg.T * cfg.E * lb
    if cfg.shared_output:
        b += cfg.T * cfg.d * ab
    return b
