"""CPU oracle of the top-k routed MoE FFN forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The product library never does, and this
package never loads the CUDA library: the two share no code.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision, serial
loops in index order); this module only compiles it with gcc, marshals numpy
arrays into its problem struct and returns numpy results.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

F32, BF16, MXFP4 = 0, 1, 2
SOFTMAX, SIGMOID = 0, 1
SILU, GELU_ERF, GELU_TANH, RELU, IDENTITY = 0, 1, 2, 3, 4
CONCAT, INTERLEAVED, UNFUSED = 0, 1, 2
GATED, PLAIN = 0, 1

_DTYPE_CODE = {"f32": F32, "bf16": BF16, "mxfp4": MXFP4}
_SCORE_CODE = {"softmax": SOFTMAX, "sigmoid": SIGMOID}
_ACT_CODE = {"silu": SILU, "gelu_erf": GELU_ERF, "gelu_tanh": GELU_TANH, "relu": RELU,
             "identity": IDENTITY}
_LAYOUT_CODE = {"concat": CONCAT, "interleaved": INTERLEAVED, "unfused": UNFUSED}
_FFN_CODE = {"gated": GATED, "plain": PLAIN}


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so (gcc, OpenMP) when stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(C.Structure):
    _fields_ = [
        ("T", C.c_int64), ("d", C.c_int64), ("F", C.c_int64), ("E", C.c_int64),
        ("k", C.c_int64), ("Fs", C.c_int64),
        ("act_dtype", C.c_int32), ("w_dtype", C.c_int32), ("logit_dtype", C.c_int32),
        ("score", C.c_int32), ("renormalize", C.c_int32),
        ("routed_scale", C.c_double),
        ("n_group", C.c_int32), ("topk_group", C.c_int32), ("weigh_inputs", C.c_int32),
        ("act", C.c_int32),
        ("alpha", C.c_double), ("beta", C.c_double), ("limit", C.c_double),
        ("gu_layout", C.c_int32), ("shared_gate", C.c_int32), ("ffn", C.c_int32),
        ("x", C.c_void_p), ("logits", C.c_void_p), ("router_bias", C.c_void_p),
        ("selection_bias", C.c_void_p),
        ("gate_up", C.c_void_p), ("gate_up_scales", C.c_void_p), ("gate_up_bias", C.c_void_p),
        ("down", C.c_void_p), ("down_scales", C.c_void_p), ("down_bias", C.c_void_p),
        ("shared_gate_up", C.c_void_p), ("shared_down", C.c_void_p),
        ("shared_gate_vec", C.c_void_p), ("shared_output", C.c_void_p),
        ("gate", C.c_void_p), ("gate_scales", C.c_void_p), ("gate_bias", C.c_void_p),
        ("router_weight", C.c_void_p),
    ]


_lib = None


def _bind(lib):
    """Declares the argument and result types of the oracle's C functions on ``lib``."""
    P = C.POINTER(_Problem)
    lib.orc_route.argtypes = [P, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
    lib.orc_route.restype = C.c_int
    lib.orc_expert.argtypes = [P, C.c_int64, C.c_void_p, C.c_void_p]
    lib.orc_expert.restype = C.c_int
    lib.orc_token.argtypes = [P, C.c_int64, C.c_void_p]
    lib.orc_token.restype = C.c_int
    lib.orc_forward.argtypes = [P, C.c_void_p, C.c_int64, C.c_void_p, C.c_int]
    lib.orc_forward.restype = C.c_int
    lib.orc_bf16.argtypes = [C.c_uint16]
    lib.orc_bf16.restype = C.c_double
    lib.orc_e2m1.argtypes = [C.c_int]
    lib.orc_e2m1.restype = C.c_double
    lib.orc_e8m0.argtypes = [C.c_int]
    lib.orc_e8m0.restype = C.c_double
    lib.orc_max_threads.restype = C.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(C.CDLL(build()))
    return _lib


def _arr(a):
    """Host array (numpy or CPU torch tensor) -> C-contiguous numpy array (bf16 as uint16 bits)."""
    if a is None:
        return None
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16)
            return a.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(a)


_TENSORS = ("x", "logits", "router_bias", "selection_bias", "gate_up", "gate_up_scales",
            "gate_up_bias", "down", "down_scales", "down_bias", "shared_gate_up", "shared_down",
            "shared_gate_vec", "shared_output", "gate", "gate_scales", "gate_bias", "router_weight")


@dataclass
class Problem:
    """One MoE forward problem on host memory, as the oracle reads it.

    ``tensors`` maps names to arrays; bf16 data may be given as torch bf16
    tensors or uint16 bit arrays.  ``cfg`` carries shapes and options with the
    attribute names of ``workloads.MoeConfig``.
    """
    cfg: object
    tensors: dict

    def __post_init__(self):
        self._keep = {n: _arr(self.tensors.get(n)) for n in _TENSORS}
        c = self.cfg
        w_dtype = c.w_dtype
        act_dtype = c.act_dtype
        p = _Problem()
        p.T, p.d, p.F, p.E, p.k, p.Fs = c.T, c.d, c.F, c.E, c.k, c.Fs
        p.act_dtype = _DTYPE_CODE[act_dtype]
        p.w_dtype = _DTYPE_CODE[w_dtype]
        p.logit_dtype = _DTYPE_CODE[c.logit_dtype]
        p.score = _SCORE_CODE[c.score]
        p.renormalize = int(c.renormalize)
        p.routed_scale = float(np.float32(c.routed_scale))
        p.n_group, p.topk_group = c.n_group, c.topk_group
        p.weigh_inputs = int(c.weigh_inputs)
        p.act = _ACT_CODE[c.act]
        p.alpha = float(np.float32(c.alpha))
        p.beta = float(np.float32(c.beta))
        p.limit = float(np.float32(c.limit))
        p.gu_layout = _LAYOUT_CODE[c.gu_layout]
        p.shared_gate = int(c.shared_gate)
        p.ffn = _FFN_CODE[getattr(c, "ffn", "gated")]
        for n in _TENSORS:
            a = self._keep[n]
            setattr(p, n, None if a is None else a.ctypes.data)
        self._p = p

    # -- calls ------------------------------------------------------------------------
    def route(self, t: int):
        """(idx[k] int32, w[k] float64, keys[E] float64, scores[E] float64) of token t."""
        lib = _load()
        k, E = self.cfg.k, self.cfg.E
        idx = np.zeros(k, np.int32)
        w = np.zeros(k, np.float64)
        keys = np.zeros(E, np.float64)
        scores = np.zeros(E, np.float64)
        rc = lib.orc_route(C.byref(self._p), t, idx.ctypes.data, w.ctypes.data,
                           keys.ctypes.data, scores.ctypes.data)
        if rc != 0:
            raise ValueError("oracle rejected the routing arguments")
        return idx, w, keys, scores

    def route_all(self):
        """Routing of every token: (idx[T,k] int32, w[T,k] float64)."""
        T, k = self.cfg.T, self.cfg.k
        idx = np.zeros((T, k), np.int32)
        w = np.zeros((T, k), np.float64)
        for t in range(T):
            idx[t], w[t], _, _ = self.route(t)
        return idx, w

    def expert(self, e: int, z):
        """One expert (e == E: the shared expert) on an input row z[d] (float64)."""
        lib = _load()
        z = np.ascontiguousarray(z, np.float64)
        out = np.zeros(self.cfg.d, np.float64)
        if lib.orc_expert(C.byref(self._p), e, z.ctypes.data, out.ctypes.data) != 0:
            raise ValueError("oracle rejected the expert arguments")
        return out

    def forward(self, tokens=None, nthreads: int = 0):
        """y[len(tokens), d] float64 for the given token indices (default: all)."""
        lib = _load()
        if tokens is None:
            tokens = np.arange(self.cfg.T, dtype=np.int64)
        tokens = np.ascontiguousarray(tokens, np.int64)
        y = np.zeros((len(tokens), self.cfg.d), np.float64)
        rc = lib.orc_forward(C.byref(self._p), tokens.ctypes.data, len(tokens), y.ctypes.data,
                             nthreads)
        if rc != 0:
            raise ValueError("oracle rejected the problem")
        return y


def decode_bf16(bits: int) -> float:
    return _load().orc_bf16(bits)


def decode_e2m1(code: int) -> float:
    return _load().orc_e2m1(code)


def decode_e8m0(s: int) -> float:
    return _load().orc_e8m0(s)


def max_threads() -> int:
    return _load().orc_max_threads()
