"""Python binding of libmoe_b200 -- the B200 top-k routed MoE FFN forward.

Argument marshalling only: every step of the forward runs in the CUDA library
(``libmoe_b200.so``, built in-tree by ``build.py``).  PyTorch supplies device
memory and streams.  There is no fallback: while the library is missing,
every entry point raises ImportError (the package itself stays importable so
that ``build.py`` can run).

Entry points mirror ``include/moe.h``: ``moe_options_init``,
``moe_workspace_size``, ``moe_forward``, ``moe_route``, ``moe_last_error``,
``moe_debug_status``, ``moe_version``; plus ``forward(...)``/``route(...)``
helpers that marshal torch tensors.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_NULL, MOE_ERR_SHAPE, MOE_ERR_DTYPE, MOE_ERR_ALIGN = 0, 1, 2, 3, 4
MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_ARG = 5, 6, 7, 8, 9
MOE_F32, MOE_BF16, MOE_MXFP4 = 0, 1, 2
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID = 0, 1
MOE_ACT_SILU, MOE_ACT_GELU_ERF, MOE_ACT_GELU_TANH, MOE_ACT_RELU, MOE_ACT_IDENTITY = 0, 1, 2, 3, 4
MOE_GU_CONCAT, MOE_GU_INTERLEAVED, MOE_GU_UNFUSED = 0, 1, 2
MOE_FFN_GATED, MOE_FFN_PLAIN = 0, 1

STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_NULL", 2: "MOE_ERR_SHAPE", 3: "MOE_ERR_DTYPE",
                4: "MOE_ERR_ALIGN", 5: "MOE_ERR_UNSUPPORTED", 6: "MOE_ERR_WORKSPACE",
                7: "MOE_ERR_CUDA", 8: "MOE_ERR_TIMEOUT", 9: "MOE_ERR_ARG"}
DTYPE_CODES = {"f32": MOE_F32, "bf16": MOE_BF16, "mxfp4": MOE_MXFP4}
SCORE_CODES = {"softmax": MOE_SCORE_SOFTMAX, "sigmoid": MOE_SCORE_SIGMOID}
ACT_CODES = {"silu": MOE_ACT_SILU, "gelu_erf": MOE_ACT_GELU_ERF, "gelu_tanh": MOE_ACT_GELU_TANH,
             "relu": MOE_ACT_RELU, "identity": MOE_ACT_IDENTITY}
LAYOUT_CODES = {"concat": MOE_GU_CONCAT, "interleaved": MOE_GU_INTERLEAVED, "unfused": MOE_GU_UNFUSED}
FFN_CODES = {"gated": MOE_FFN_GATED, "plain": MOE_FFN_PLAIN}


class moe_shape(C.Structure):
    _fields_ = [("T", C.c_int64), ("d", C.c_int64), ("F", C.c_int64), ("E", C.c_int64),
                ("k", C.c_int64), ("Fs", C.c_int64), ("act_dtype", C.c_int32),
                ("w_dtype", C.c_int32), ("logit_dtype", C.c_int32), ("reserved", C.c_int32)]


class moe_options(C.Structure):
    _fields_ = [("score", C.c_int32), ("renormalize", C.c_int32), ("routed_scale", C.c_float),
                ("n_group", C.c_int32), ("topk_group", C.c_int32), ("weigh_inputs", C.c_int32),
                ("act", C.c_int32), ("alpha", C.c_float), ("beta", C.c_float),
                ("limit", C.c_float), ("gu_layout", C.c_int32), ("shared_gate", C.c_int32),
                ("ffn", C.c_int32)]


class moe_tensors(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in (
        "x", "router_logits", "router_bias", "selection_bias", "gate_up", "gate_up_scales",
        "gate_up_bias", "down", "down_scales", "down_bias", "shared_gate_up", "shared_down",
        "shared_gate_vec", "shared_output", "y", "topk_idx", "topk_w", "gate", "gate_scales",
        "gate_bias", "router_weight", "logits_out")]


_P = C.POINTER
MOE_STAGE_EVENTS = 7
STAGES = ("route", "sort", "gather", "gate_up", "down", "combine")


def _bind(lib: C.CDLL) -> C.CDLL:
    """Declares the argument and result types of every entry point of include/moe.h."""
    lib.moe_options_init.argtypes = [_P(moe_options)]
    lib.moe_options_init.restype = None
    lib.moe_workspace_size.argtypes = [_P(moe_shape), _P(moe_options)]
    lib.moe_workspace_size.restype = C.c_size_t
    for fn in (lib.moe_forward, lib.moe_route):
        fn.argtypes = [_P(moe_shape), _P(moe_options), _P(moe_tensors), C.c_void_p, C.c_size_t,
                       C.c_void_p]
        fn.restype = C.c_int
    lib.moe_forward_events.argtypes = [_P(moe_shape), _P(moe_options), _P(moe_tensors), C.c_void_p,
                                       C.c_size_t, C.c_void_p, _P(C.c_void_p), C.c_int]
    lib.moe_forward_events.restype = C.c_int
    lib.moe_forward_noalloc.argtypes = [_P(moe_shape), _P(moe_options), _P(moe_tensors), C.c_void_p]
    lib.moe_forward_noalloc.restype = C.c_int
    lib.moe_noalloc_debug_status.argtypes = [C.c_void_p]
    lib.moe_noalloc_debug_status.restype = C.c_int
    lib.moe_noalloc_workspace_bytes.argtypes = []
    lib.moe_noalloc_workspace_bytes.restype = C.c_size_t
    lib.moe_permute.argtypes = [_P(moe_shape), _P(moe_options), C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_size_t,
                                C.c_void_p]
    lib.moe_permute.restype = C.c_int
    lib.moe_experts_forward.argtypes = [_P(moe_shape), _P(moe_options), _P(moe_tensors), C.c_void_p, C.c_void_p,
                                        C.c_void_p, C.c_size_t, C.c_void_p]
    lib.moe_experts_forward.restype = C.c_int
    lib.moe_combine.argtypes = [_P(moe_shape), C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p,
                                C.c_void_p]
    lib.moe_combine.restype = C.c_int
    lib.moe_forward_kernel_count.argtypes = [_P(moe_shape), _P(moe_options)]
    lib.moe_forward_kernel_count.restype = C.c_int
    lib.moe_forward_split_k.argtypes = [_P(moe_shape), _P(moe_options), _P(C.c_int), _P(C.c_int)]
    lib.moe_forward_split_k.restype = C.c_int
    lib.moe_forward_fused_gemms.argtypes = [_P(moe_shape), _P(moe_options)]
    lib.moe_forward_fused_gemms.restype = C.c_int
    lib.moe_last_error.argtypes = []
    lib.moe_last_error.restype = C.c_char_p
    lib.moe_debug_status.argtypes = [C.c_void_p, C.c_void_p]
    lib.moe_debug_status.restype = C.c_int
    lib.moe_version.argtypes = []
    lib.moe_version.restype = C.c_char_p
    return lib


class _UnbuiltLibrary:
    """Stands in for the CUDA library until its first use.  The package imports
    without loading it, so that its build step can run (and replace a library built
    from older sources); the first entry point called loads and binds it, raising
    ImportError while it is missing or lacks an entry point of these bindings.
    There is no fallback: nothing here computes without the CUDA library."""

    def __getattr__(self, name):
        global _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python "
                              f"{os.path.join(_HERE, 'build.py')}` (nvcc, sm_100a)")
        handle = C.CDLL(LIB_PATH)
        try:
            lib = _bind(handle)
        except AttributeError as e:
            import _ctypes
            _ctypes.dlclose(handle._handle)  # a rebuilt library then loads afresh
            raise ImportError(f"{LIB_PATH} was built from older sources ({e}): rebuild it with "
                              f"`python {os.path.join(_HERE, 'build.py')}`") from None
        _lib = lib
        return getattr(_lib, name)


_lib = _UnbuiltLibrary()

EXPORTED = ("moe_options_init", "moe_workspace_size", "moe_forward", "moe_route",
            "moe_forward_events", "moe_forward_noalloc", "moe_noalloc_debug_status",
            "moe_noalloc_workspace_bytes", "moe_forward_kernel_count", "moe_forward_split_k",
            "moe_forward_fused_gemms", "moe_last_error", "moe_debug_status", "moe_version",
            "moe_permute", "moe_experts_forward", "moe_combine")


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


# ---------------------------------------------------------------------- raw entry points
def moe_options_init() -> moe_options:
    o = moe_options()
    _lib.moe_options_init(C.byref(o))
    return o


def moe_workspace_size(shape: moe_shape, opts: moe_options) -> int:
    return _lib.moe_workspace_size(C.byref(shape), C.byref(opts))


def moe_forward(shape, opts, tensors, workspace: int, workspace_bytes: int, stream: int) -> int:
    return _lib.moe_forward(C.byref(shape), C.byref(opts), C.byref(tensors), workspace,
                            workspace_bytes, stream)


def moe_route(shape, opts, tensors, workspace: int, workspace_bytes: int, stream: int) -> int:
    return _lib.moe_route(C.byref(shape), C.byref(opts), C.byref(tensors), workspace,
                          workspace_bytes, stream)


def moe_forward_events(shape, opts, tensors, workspace: int, workspace_bytes: int, stream: int,
                       events) -> int:
    """moe_forward recording raw cudaEvent_t handles (ints) at the stage boundaries."""
    arr = (C.c_void_p * len(events))(*events)
    return _lib.moe_forward_events(C.byref(shape), C.byref(opts), C.byref(tensors), workspace,
                                   workspace_bytes, stream, arr, len(events))


def moe_forward_noalloc(shape, opts, tensors, stream: int) -> int:
    """moe_forward on the library's static scratch array (no workspace argument)."""
    return _lib.moe_forward_noalloc(C.byref(shape), C.byref(opts), C.byref(tensors), stream)


def moe_noalloc_debug_status(stream: int) -> int:
    """Device status word of the last moe_forward_noalloc on the current context."""
    return _lib.moe_noalloc_debug_status(stream)


def moe_noalloc_workspace_bytes() -> int:
    """Size of the library's static scratch array (read from the library)."""
    return _lib.moe_noalloc_workspace_bytes()


def moe_permute(shape, opts, idx: int, w: int, x: int, x_perm: int, row_expert: int, row_w: int,
                expert_counts: int, pos: int, experts_per_rank: int, workspace: int, workspace_bytes: int,
                stream: int) -> int:
    return _lib.moe_permute(C.byref(shape), C.byref(opts), idx, w, x, x_perm, row_expert, row_w, expert_counts,
                            pos, experts_per_rank, workspace, workspace_bytes, stream)


def moe_experts_forward(shape, opts, tensors, row_expert: int, row_w: int, workspace: int,
                        workspace_bytes: int, stream: int) -> int:
    return _lib.moe_experts_forward(C.byref(shape), C.byref(opts), C.byref(tensors), row_expert, row_w,
                                    workspace, workspace_bytes, stream)


def moe_combine(shape, pos: int, Y: int, rows: int, shared_output: int, y: int, stream: int) -> int:
    return _lib.moe_combine(C.byref(shape), pos, Y, rows, shared_output, y, stream)


def moe_forward_kernel_count(shape, opts) -> int:
    return _lib.moe_forward_kernel_count(C.byref(shape), C.byref(opts))


def moe_forward_split_k(shape, opts):
    """(gate_up splits, down splits) of the forward's GEMMs; raises MoeError on bad arguments."""
    sg, sd = C.c_int(0), C.c_int(0)
    rc = _lib.moe_forward_split_k(C.byref(shape), C.byref(opts), C.byref(sg), C.byref(sd))
    if rc != 0:
        raise MoeError(rc, moe_last_error())
    return sg.value, sd.value


def moe_forward_fused_gemms(shape, opts) -> int:
    return _lib.moe_forward_fused_gemms(C.byref(shape), C.byref(opts))


def moe_last_error() -> str:
    return _lib.moe_last_error().decode()


def moe_debug_status(workspace: int, stream: int) -> int:
    return _lib.moe_debug_status(workspace, stream)


def moe_version() -> str:
    return _lib.moe_version().decode()


# ---------------------------------------------------------------------- marshalling helpers
def make_shape(T, d, F, E, k, Fs=0, act_dtype="bf16", w_dtype="bf16", logit_dtype="bf16"):
    return moe_shape(T, d, F, E, k, Fs, DTYPE_CODES[act_dtype], DTYPE_CODES[w_dtype],
                     DTYPE_CODES[logit_dtype], 0)


def make_options(score="softmax", renormalize=False, routed_scale=1.0, n_group=0, topk_group=0,
                 weigh_inputs=False, act="silu", alpha=1.0, beta=0.0, limit=0.0,
                 gu_layout="concat", shared_gate=False, ffn="gated") -> moe_options:
    o = moe_options_init()
    o.score = SCORE_CODES[score]
    o.renormalize = int(renormalize)
    o.routed_scale = routed_scale
    o.n_group, o.topk_group = n_group, topk_group
    o.weigh_inputs = int(weigh_inputs)
    o.act = ACT_CODES[act]
    o.alpha, o.beta, o.limit = alpha, beta, limit
    o.gu_layout = LAYOUT_CODES[gu_layout]
    o.shared_gate = int(shared_gate)
    o.ffn = FFN_CODES[ffn]
    return o


def shape_of(cfg) -> moe_shape:
    """moe_shape from any object with the attributes of a workload config."""
    return make_shape(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.Fs, cfg.act_dtype, cfg.w_dtype,
                      cfg.logit_dtype)


def options_of(cfg) -> moe_options:
    return make_options(cfg.score, cfg.renormalize, cfg.routed_scale, cfg.n_group,
                        cfg.topk_group, cfg.weigh_inputs, cfg.act, cfg.alpha, cfg.beta,
                        cfg.limit, cfg.gu_layout, cfg.shared_gate, getattr(cfg, "ffn", "gated"))


def _ptr(t):
    return None if t is None else t.data_ptr()


def tensors_of(inputs: dict, y=None, topk_idx=None, topk_w=None, logits_out=None) -> moe_tensors:
    """moe_tensors from a dict of device tensors (keys as in moe.h)."""
    t = moe_tensors()
    for name in ("x", "router_bias", "selection_bias", "gate_up", "gate_up_scales",
                 "gate_up_bias", "down", "down_scales", "down_bias", "shared_gate_up",
                 "shared_down", "shared_gate_vec", "shared_output", "gate", "gate_scales",
                 "gate_bias", "router_weight"):
        setattr(t, name, _ptr(inputs.get(name)))
    t.router_logits = _ptr(inputs.get("logits", inputs.get("router_logits")))
    t.y, t.topk_idx, t.topk_w = _ptr(y), _ptr(topk_idx), _ptr(topk_w)
    t.logits_out = _ptr(logits_out)
    return t


def _check(rc: int):
    if rc != MOE_OK:
        raise MoeError(rc, moe_last_error())


class Workspace:
    """Device workspace sized by moe_workspace_size (allocated by torch, not the library)."""

    def __init__(self, nbytes: int, device="cuda"):
        import torch
        self.nbytes = int(nbytes)
        self.buf = torch.empty(max(self.nbytes, 256), dtype=torch.uint8, device=device)

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()


def forward(cfg, inputs: dict, y=None, workspace: Workspace | None = None, stream=None,
            topk_idx=None, topk_w=None, logits_out=None):
    """Run moe_forward on device tensors; returns y [T, d] (allocated by torch if None)."""
    import torch
    x = inputs["x"]
    shape, opts = shape_of(cfg), options_of(cfg)
    if y is None:
        y = torch.empty_like(x)
    if workspace is None:
        workspace = Workspace(moe_workspace_size(shape, opts), x.device)
    st = (stream if stream is not None else torch.cuda.current_stream(x.device)).cuda_stream
    tens = tensors_of(inputs, y, topk_idx, topk_w, logits_out)
    _check(moe_forward(shape, opts, tens, workspace.ptr, workspace.nbytes, st))
    return y


def route(cfg, inputs: dict, workspace: Workspace | None = None, stream=None):
    """Run moe_route; returns (topk_idx [T, k] int32, topk_w [T, k] fp32)."""
    import torch
    logits = inputs["logits"] if inputs.get("logits") is not None else inputs["x"]
    shape, opts = shape_of(cfg), options_of(cfg)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=logits.device)
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=logits.device)
    if workspace is None:
        workspace = Workspace(moe_workspace_size(shape, opts), logits.device)
    st = (stream if stream is not None else torch.cuda.current_stream(logits.device)).cuda_stream
    _check(moe_route(shape, opts, tensors_of(inputs, None, idx, w), workspace.ptr,
                     workspace.nbytes, st))
    return idx, w
