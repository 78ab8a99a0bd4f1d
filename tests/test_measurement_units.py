"""The algorithmic units behind every roofline fraction `bench.py` reports, checked
against figures worked out by hand from the workload shapes (CPU only).

FLOPs of a forward = 2 * (T*k routed rows) * 3*d*F + 2 * T * 3*d*Fs; bytes = the
touched experts' weights (+ MXFP4 scales, + expert biases) + shared weights + x,
logits and y.
"""
import os

import pytest

import bench
from workloads import CONFIGS, algorithmic_bytes, flops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# name: (experts touched, FLOPs, bytes), each worked out by hand:
HAND = {
    # 2*128*3*128*256; 8 experts * 3*128*256 * 4 B + x, y (64*128*4 each) + logits 64*8*4
    "tiny_fp32": (8, 25_165_824, 8 * 3 * 128 * 256 * 4 + 2 * 64 * 128 * 4 + 64 * 8 * 4),
    # 2*8192*3*4096*14336; 8 * 3*4096*14336 * 2 B = 2.819 GB + x, y 2 * 4096*4096*2 + logits
    "mixtral_bf16": (8, 2.886e12, 8 * 3 * 4096 * 14336 * 2 + 2 * 4096 * 4096 * 2 + 4096 * 8 * 2),
    # 2*8192*3*2880^2; per expert 3*2880^2/2 codes + /32 scales + (2*2880+2880)*2 bias bytes
    "gptoss_mxfp4": (32, 4.0769e11, 32 * (3 * 2880 * 2880 * (1 / 2 + 1 / 32) + 3 * 2880 * 2)
                     + 2 * 2048 * 2880 * 2 + 2048 * 32 * 2),
    # 2*65536*3*7168*2048 + 2*8192*3*7168*2048; (256 routed + 1 shared) * 3*7168*2048*2 B
    "deepseek_bf16": (256, 6.494e12, 257 * 3 * 7168 * 2048 * 2 + 2 * 8192 * 7168 * 2 + 8192 * 256 * 2),
    # 2*8*3*4096*1536; 8 experts * 37.75 MB + x, y, logits of one token
    "decode_T1": (8, 3.0199e8, 8 * 3 * 4096 * 1536 * 2 + 2 * 4096 * 2 + 128 * 2),
}


@pytest.mark.parametrize("name", list(HAND))
def test_layer_flops_and_bytes(name):
    cfg = CONFIGS[name]
    distinct, f, b = HAND[name]
    assert flops(cfg) == pytest.approx(f, rel=1e-4)
    assert algorithmic_bytes(cfg, distinct) == pytest.approx(b, rel=1e-9)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_stage_flops_add_up_to_the_layer(name):
    cfg = CONFIGS[name]
    m = bench.stage_model(cfg, cfg.E)
    assert m["gate_up"]["flops"] + m["down"]["flops"] == flops(cfg)
    assert m["gate_up"]["flops"] == 2 * m["down"]["flops"]  # 2F output columns against F of K


def test_stage_bytes_count_each_weight_once():
    cfg = CONFIGS["mixtral_bf16"]
    m = bench.stage_model(cfg, 8)
    R = cfg.T * cfg.k
    w = 8 * 3 * cfg.d * cfg.F * 2
    # gate_up reads 2/3 of the weights, the gathered rows (d) and writes h (F); down the rest
    assert m["gate_up"]["bytes"] == 2 * w / 3 + R * (cfg.d + cfg.F) * 2
    assert m["down"]["bytes"] == w / 3 + R * (cfg.F + cfg.d) * 2


def test_traffic_figures_follow_their_kernel_sources(monkeypatch):
    # each stored DRAM figure is reported only while its kernel's sources are unchanged
    for (wl, st), (nbytes, kfile, h) in bench.NCU_TRAFFIC.items():
        assert bench.ncu_traffic(wl, st) == (nbytes if h == bench.kernel_sources_hash(kfile) else None)
    key = ("mixtral_bf16", "gate_up")
    nbytes, kfile, _ = bench.NCU_TRAFFIC[key]
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, (nbytes, kfile, "0" * 12))
    assert bench.ncu_traffic(*key) is None
    assert bench.ncu_traffic("mixtral_bf16", "combine") is None


def test_comment_edits_leave_the_code_hash_alone():
    a = b"int f(int x) {  // doubles\n  return 2 * x; /* the\n body */\n}\n"
    b = b"int f(int x) {\n\n  return 2 * x;\n}  // changed\n"
    assert bench._code_of(a) == bench._code_of(b)
    assert bench._code_of(a) != bench._code_of(a.replace(b"2 * x", b"3 * x"))


def test_kernel_hash_covers_included_headers_only():
    import hashlib
    csrc = os.path.join(ROOT, "mixture_experts_ffn_10_b200", "csrc")
    files = ["common.cuh", "epilogue.cuh", "gemm_tcs.cu", "sm100.cuh", "tmap.cuh"]
    h = hashlib.sha256()
    for f in [os.path.join(csrc, f) for f in files] + [os.path.join(ROOT, "include", "moe.h")]:
        h.update(os.path.basename(f).encode())
        h.update(bench._code_of(open(f, "rb").read()))
    assert bench.kernel_sources_hash("gemm_tcs.cu") == h.hexdigest()[:12]


def test_traffic_only_for_the_default_kernels(monkeypatch):
    """An environment variable that overrides the kernel choice detaches the stored ncu
    traffic figures (they were captured with the library's own choice)."""
    import bench
    assert bench.default_kernels()
    for v in bench.KERNEL_CHOICE_VARS:
        monkeypatch.setenv(v, "1")
        assert not bench.default_kernels()
        monkeypatch.delenv(v)
    assert bench.default_kernels()
