"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/moe.h declares, and rejects bad arguments on the host before any launch."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moe():
    from mixture_experts_ffn_10_b200 import build
    build.build()
    import mixture_experts_ffn_10_b200 as m
    return m


def _declared():
    src = ""
    for h in ("moe.h", "moe_ep.h"):
        with open(os.path.join(ROOT, "include", h)) as f:
            src += f.read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    assert _declared() == sorted(["moe_options_init", "moe_workspace_size", "moe_forward",
                                  "moe_route", "moe_forward_events", "moe_forward_noalloc",
                                  "moe_noalloc_debug_status", "moe_noalloc_workspace_bytes",
                                  "moe_forward_kernel_count", "moe_forward_split_k",
                                  "moe_forward_fused_gemms", "moe_last_error", "moe_debug_status",
                                  "moe_version", "moe_permute", "moe_experts_forward", "moe_combine"])


def test_static_scratch_size_matches_the_header(moe):
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        m = re.search(r"#define MOE_NOALLOC_WORKSPACE_BYTES \((\d+)u << (\d+)\)", f.read())
    assert m, "MOE_NOALLOC_WORKSPACE_BYTES not found in the header"
    assert moe.moe_noalloc_workspace_bytes() == int(m.group(1)) << int(m.group(2))


def test_library_exports_every_declared_symbol(moe):
    lib = C.CDLL(moe.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(moe.EXPORTED) == set(_declared())


def test_struct_sizes_match_the_header(moe):
    # int64 x 6 + int32 x 4; 13 x 4-byte fields; 22 pointers
    assert C.sizeof(moe.moe_shape) == 64
    assert C.sizeof(moe.moe_options) == 52
    assert C.sizeof(moe.moe_tensors) == 22 * 8


def test_options_defaults(moe):
    o = moe.moe_options_init()
    assert (o.score, o.renormalize, o.routed_scale, o.n_group, o.weigh_inputs) == (0, 0, 1.0, 0, 0)
    assert (o.act, o.alpha, o.beta, o.limit, o.gu_layout, o.shared_gate) == (0, 1.0, 0.0, 0.0, 0, 0)
    assert moe.moe_version().startswith("moe_b200")


def _valid(moe, **kw):
    args = dict(T=64, d=128, F=256, E=8, k=2, Fs=0, act_dtype="bf16", w_dtype="bf16",
                logit_dtype="bf16")
    args.update(kw)
    return moe.make_shape(**args)


def test_workspace_size_grows_with_tokens(moe):
    o = moe.make_options(renormalize=True)
    a = moe.moe_workspace_size(_valid(moe, T=64), o)
    b = moe.moe_workspace_size(_valid(moe, T=128), o)
    assert 0 < a < b and a % 256 == 0
    assert moe.moe_workspace_size(_valid(moe, k=9), o) == 0
    assert "k" in moe.moe_last_error()


FAKE = 1 << 20  # a non-NULL, 256-aligned address: validation never dereferences it


def _tensors(moe, **kw):
    t = moe.moe_tensors()
    for n in ("x", "router_logits", "gate_up", "down", "y"):
        setattr(t, n, FAKE)
    for n, v in kw.items():
        setattr(t, n, v)
    return t


@pytest.mark.parametrize("shape_kw,opt_kw,tens_kw,code", [
    (dict(k=0), {}, {}, 2),
    (dict(k=9), {}, {}, 2),
    (dict(d=12), {}, {}, 2),
    (dict(T=-1), {}, {}, 2),
    (dict(act_dtype="f32", w_dtype="bf16"), {}, {}, 3),
    (dict(E=2048, k=2), {}, {}, 5),
    (dict(k=33, E=64), {}, {}, 5),
    (dict(w_dtype="mxfp4", d=80), {}, {}, 2),
    ({}, dict(n_group=3, topk_group=1), {}, 9),
    ({}, dict(n_group=4, topk_group=5), {}, 9),
    (dict(E=8, k=4), dict(n_group=4, topk_group=1), {}, 9),
    ({}, dict(limit=-1.0), {}, 9),
    ({}, dict(routed_scale=float("inf")), {}, 9),
    ({}, dict(shared_gate=True), {}, 9),
    ({}, {}, dict(x=None), 1),
    ({}, {}, dict(router_logits=None), 1),
    ({}, {}, dict(gate_up=FAKE + 8), 4),
    ({}, {}, dict(y=FAKE), 9),
    (dict(Fs=64), {}, {}, 1),
    ({}, dict(gu_layout="unfused"), {}, 1),                           # no gate stack
    ({}, dict(gu_layout="unfused", ffn="plain"), dict(gate=FAKE), 9),  # unfused needs a gated FFN
    ({}, {}, dict(gate=FAKE), 9),                                      # gate given to a fused layout
    (dict(w_dtype="mxfp4"), dict(gu_layout="unfused"),
     dict(gate=FAKE, gate_up_scales=FAKE, down_scales=FAKE), 1),     # no gate_scales
    ({}, {}, dict(router_weight=FAKE), 9),                             # logits and router weight
    ({}, {}, dict(router_logits=None, router_weight=FAKE, x=None), 1),
    ({}, {}, dict(logits_out=FAKE), 9),                                # logits_out without router weight
    ({}, {}, dict(gate=FAKE + 8), 9),
])
def test_validation_rejects_before_launch(moe, shape_kw, opt_kw, tens_kw, code):
    s = _valid(moe, **shape_kw)
    o = moe.make_options(**opt_kw)
    t = _tensors(moe, **tens_kw)
    if tens_kw.get("y") == FAKE:
        t.x = FAKE  # y aliases x
    else:
        t.y = 2 * FAKE
    rc = moe.moe_forward(s, o, t, FAKE, 1 << 40, None)
    assert rc == code, (rc, moe.moe_last_error())
    assert moe.moe_last_error()


def test_workspace_checks(moe):
    s, o = _valid(moe), moe.make_options()
    t = _tensors(moe)
    t.y = FAKE * 2
    need = moe.moe_workspace_size(s, o)
    assert moe.moe_forward(s, o, t, None, need, None) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_forward(s, o, t, FAKE, need - 1, None) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_forward(s, o, t, FAKE + 16, need, None) == moe.MOE_ERR_WORKSPACE


def test_zero_tokens_is_a_no_op(moe):
    s, o = _valid(moe, T=0), moe.make_options()
    t = _tensors(moe)
    t.y = FAKE * 2
    assert moe.moe_forward(s, o, t, FAKE, moe.moe_workspace_size(s, o), None) == moe.MOE_OK


def test_route_needs_outputs(moe):
    s, o = _valid(moe), moe.make_options()
    t = moe.moe_tensors()
    t.router_logits = FAKE
    assert moe.moe_route(s, o, t, FAKE, 1 << 40, None) == moe.MOE_ERR_NULL


def test_binding_without_its_library_imports_but_every_entry_point_raises(tmp_path):
    """A fresh checkout has no libmoe_b200.so: the package must import (its build
    step lives inside it) and each entry point must fail loudly, never compute."""
    import shutil
    import subprocess
    import sys

    pkg = tmp_path / "mixture_experts_ffn_10_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "mixture_experts_ffn_10_b200", "__init__.py"), pkg / "__init__.py")
    code = (
        "import mixture_experts_ffn_10_b200 as m\n"
        "for call in (m.moe_version, m.moe_options_init, lambda: m.moe_last_error()):\n"
        "    try:\n"
        "        call()\n"
        "    except ImportError as e:\n"
        "        assert 'is missing' in str(e)\n"
        "    else:\n"
        "        raise SystemExit('entry point ran without the library')\n"
        "print('ok')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr


@pytest.mark.parametrize("name,count", [
    ("tiny_fp32", 6), ("decode_T1", 4), ("decode_T8", 4), ("decode_T64", 4), ("decode_T256", 8),
    ("mixtral_bf16", 8), ("gptoss_mxfp4", 8), ("deepseek_bf16", 8)])
def test_kernel_count_of_each_workload(moe, name, count):
    """The launch plan on a 148-SM part (what the host assumes without a GPU): route,
    sort (one kernel for a single 64-token chunk, else histogram + scan + scatter),
    gather (not for bf16 batches of at most 64 tokens, whose gate_up reads x in
    place), gate_up, down (one launch with gate_up for those batches), combine.
    Split-K adds no launch: the last split of a tile region reduces it."""
    from workloads import CONFIGS
    cfg = CONFIGS[name]
    assert moe.moe_forward_kernel_count(moe.shape_of(cfg), moe.options_of(cfg)) == count


@pytest.mark.parametrize("name,fused", [
    ("tiny_fp32", 0), ("decode_T1", 1), ("decode_T8", 1), ("decode_T64", 1), ("decode_T256", 0),
    ("mixtral_bf16", 0), ("gptoss_mxfp4", 0), ("deepseek_bf16", 0)])
def test_fused_gemms_for_small_bf16_batches(moe, name, fused, monkeypatch):
    """1: gate_up and down in one launch (T <= 64), 0: separate launches;
    MOE_B200_FUSED_FFN=0 steps down (2, the few-token kernel, is opt-in)."""
    from workloads import CONFIGS
    cfg = CONFIGS[name]
    shape, opts = moe.shape_of(cfg), moe.options_of(cfg)
    assert moe.moe_forward_fused_gemms(shape, opts) == fused
    monkeypatch.setenv("MOE_B200_GEMV", "0")
    assert moe.moe_forward_fused_gemms(shape, opts) == min(fused, 1)
    assert moe.moe_forward_kernel_count(shape, opts) == (4 if fused else moe.moe_forward_kernel_count(shape, opts))
    monkeypatch.setenv("MOE_B200_FUSED_FFN", "0")
    assert moe.moe_forward_fused_gemms(shape, opts) == 0
    assert moe.moe_forward_kernel_count(shape, opts) == (5 if fused else moe.moe_forward_kernel_count(shape, opts))


@pytest.mark.parametrize("T,gemv", [(1, True), (4, True), (5, False)])
def test_few_token_kernel_limits(moe, T, gemv, monkeypatch):
    """The few-token kernel (opt-in: MOE_B200_GEMV=N, N <= 4 tokens) serves bf16
    weights, E <= 256 and d, F, Fs in whole 64-element blocks; forced CTA-pair GEMMs
    keep their kernels."""
    o = moe.make_options()
    sh = moe.make_shape(T=T, d=4096, F=1536, E=128, k=8)
    assert moe.moe_forward_fused_gemms(sh, o) != 2  # off by default
    monkeypatch.setenv("MOE_B200_GEMV", "4")
    assert (moe.moe_forward_fused_gemms(sh, o) == 2) == gemv
    assert (moe.moe_forward_kernel_count(sh, o) == 1) == gemv
    assert moe.moe_forward_fused_gemms(moe.make_shape(T=T, d=4096, F=1536, E=300, k=8), o) != 2
    assert moe.moe_forward_fused_gemms(moe.make_shape(T=T, d=512, F=256, E=32, k=4, w_dtype="mxfp4"), o) != 2
    assert moe.moe_forward_fused_gemms(moe.make_shape(T=T, d=200, F=256, E=32, k=4), o) != 2  # 64-element blocks
    assert moe.moe_forward_fused_gemms(moe.make_shape(T=T, d=512, F=256, E=32, k=4, Fs=96), o) != 2
    monkeypatch.setenv("MOE_B200_GEMV", "2")
    assert (moe.moe_forward_fused_gemms(sh, o) == 2) == (T <= 2)
    monkeypatch.setenv("MOE_B200_GEMV", "4")
    monkeypatch.setenv("MOE_B200_PAIR_GEMM", "1")
    assert moe.moe_forward_fused_gemms(sh, o) != 2


def test_split_k_choice_follows_the_cost_model(moe):
    """choose_splits: cost = waves * (k-blocks per unit + 2) + 4 for the read-back of
    the partials.  T=1, E=8, k=1, d=4096, F=1024: gate_up has 8 tiles x 64 k-blocks ->
    8 splits (one wave of 64 units of 8 k-blocks: cost 14 against 66); down has 16
    tiles x 16 k-blocks -> 8 splits (cost 8 against 18).  T=65 (two sort chunks):
    gate_up 64 tiles -> 2 splits (cost 38; 4 splits cost 40), down 128 tiles -> no
    split (18 against 24).  Decode T=1 (E=128, k=8, d=4096, F=1536): gate_up 96 tiles x
    64 k-blocks -> 3 splits (2 waves of 22: cost 52 against 66), down 128 tiles x 24 ->
    none (26 against 32)."""
    o = moe.make_options()
    assert moe.moe_forward_split_k(moe.make_shape(T=1, d=4096, F=1024, E=8, k=1), o) == (8, 8)
    assert moe.moe_forward_split_k(moe.make_shape(T=65, d=4096, F=1024, E=8, k=1), o) == (2, 1)
    assert moe.moe_forward_split_k(moe.make_shape(T=1, d=4096, F=1536, E=128, k=8), o) == (3, 1)
    # fp32 problems run the SIMT GEMMs, which never split K
    f32 = moe.make_shape(T=1, d=4096, F=1024, E=8, k=1, act_dtype="f32", w_dtype="f32", logit_dtype="f32")
    assert moe.moe_forward_split_k(f32, o) == (1, 1)
    assert moe.moe_forward_kernel_count(f32, o) == 6
    with pytest.raises(moe.MoeError):
        moe.moe_forward_split_k(moe.make_shape(T=1, d=4096, F=1024, E=8, k=0), o)


def test_expert_parallel_entry_points_validate_before_launch(moe):
    """moe_permute, moe_experts_forward and moe_combine reject bad arguments on the host
    (no device work): experts_per_rank must divide E; rows arriving with their expert
    take k = 1, no shared expert and no router inputs; moe_combine checks its shape."""
    s, o = _valid(moe), moe.make_options()
    need = moe.moe_workspace_size(s, o)
    args = [FAKE] * 8
    assert moe.moe_permute(s, o, *args, 3, FAKE, need, None) == moe.MOE_ERR_ARG  # E = 8
    assert moe.moe_permute(s, o, *args, -1, FAKE, need, None) == moe.MOE_ERR_ARG
    bad = list(args)
    bad[2] = None  # x
    assert moe.moe_permute(s, o, *bad, 4, FAKE, need, None) == moe.MOE_ERR_NULL
    bad = list(args)
    bad[3] = FAKE + 8  # x_perm misaligned
    assert moe.moe_permute(s, o, *bad, 4, FAKE, need, None) == moe.MOE_ERR_ALIGN
    assert moe.moe_permute(s, o, *args, 4, FAKE, need - 1, None) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_permute(_valid(moe, T=0), o, *args, 4, FAKE, need, None) == moe.MOE_OK

    t = _tensors(moe)
    t.router_logits = None
    t.y = 2 * FAKE
    s1 = _valid(moe, k=1)
    need1 = moe.moe_workspace_size(s1, o)
    assert moe.moe_experts_forward(s, o, t, FAKE, FAKE, FAKE, need, None) == moe.MOE_ERR_SHAPE  # k = 2
    assert moe.moe_experts_forward(_valid(moe, k=1, Fs=64), o, t, FAKE, FAKE, FAKE, need1, None) == \
        moe.MOE_ERR_UNSUPPORTED
    assert moe.moe_experts_forward(s1, o, t, None, FAKE, FAKE, need1, None) == moe.MOE_ERR_NULL
    t.router_logits = FAKE
    assert moe.moe_experts_forward(s1, o, t, FAKE, FAKE, FAKE, need1, None) == moe.MOE_ERR_ARG
    t.router_logits = None
    t.topk_idx = FAKE
    assert moe.moe_experts_forward(s1, o, t, FAKE, FAKE, FAKE, need1, None) == moe.MOE_ERR_ARG

    assert moe.moe_combine(s, FAKE, FAKE, -1, None, 2 * FAKE, None) == moe.MOE_ERR_SHAPE
    assert moe.moe_combine(s, None, FAKE, 16, None, 2 * FAKE, None) == moe.MOE_ERR_NULL
    assert moe.moe_combine(s, FAKE, FAKE, 16, None, FAKE, None) == moe.MOE_ERR_ARG  # y aliases Y
    assert moe.moe_combine(s, FAKE, FAKE + 8, 16, None, 2 * FAKE, None) == moe.MOE_ERR_ALIGN
    assert moe.moe_combine(_valid(moe, T=0), FAKE, FAKE, 16, None, 2 * FAKE, None) == moe.MOE_OK
