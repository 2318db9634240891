"""CPU oracle of the fused MoE layer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this package.  The product library never calls it, and it
shares no code with the CUDA path: ``moe_oracle.c`` is plain single-threaded C in
FP64 with the rounding points listed in its header.

Functions take numpy arrays (BF16 as ``uint16`` bit patterns, FP32 as ``float32``).
Every function pins to something other than itself in ``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SCORE = {"softmax": 0, "sigmoid": 1}
ACT = {"swiglu": 0, "relu2": 1}


def build(force: bool = False) -> str:
    """Compile ``moe_oracle.c`` with gcc (strict IEEE: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("T", "H", "I", "E", "K", "act", "score", "renorm", "I_shared")] + [
        ("router_w", ctypes.c_void_p), ("router_logits", ctypes.c_void_p), ("bias", ctypes.c_void_p),
        ("w13", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("ws13", ctypes.c_void_p), ("ws2", ctypes.c_void_p),
        ("routed_scale", ctypes.c_double), ("shared_gate", ctypes.c_void_p), ("shared_out", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_bf16_to_double.restype = ctypes.c_double
        _lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        _lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        _lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        _lib.oracle_sigmoid_f32.restype = ctypes.c_float
        _lib.oracle_sigmoid_f32.argtypes = [ctypes.c_float]
        vp, ci = ctypes.c_void_p, ctypes.c_int
        _lib.oracle_router_logits.argtypes = [vp, vp, ci, ci, ci, vp]
        _lib.oracle_topk.argtypes = [vp, ci, ci, ci, ci, ci, vp, ci, vp, vp, vp]
        _lib.oracle_topk.restype = ci
        _lib.oracle_permute.argtypes = [vp, ci, ci, ci, vp, vp, vp]
        _lib.oracle_permute.restype = ci
        _lib.oracle_forward_rows.argtypes = [ctypes.POINTER(_Layer), vp, vp, ci, vp, vp, vp, vp]
        _lib.oracle_forward_rows.restype = ci
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(bits)


def double_to_bf16(v: float) -> int:
    return lib().oracle_double_to_bf16(v)


def sigmoid_f32(l: float) -> float:
    return lib().oracle_sigmoid_f32(l)


def router_logits(x_bits: np.ndarray, wr_bits: np.ndarray) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    wr = _c(wr_bits, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float32)
    lib().oracle_router_logits(_p(x), _p(wr), T, H, E, _p(out))
    return out


def topk(logits: np.ndarray, K: int, score: str, bias=None, renorm: bool = True,
         logits_bf16: bool = False):
    """Router top-k.  ``logits``: [M,E] float32, or uint16 BF16 bits with ``logits_bf16``."""
    lg = _c(logits, np.uint16 if logits_bf16 else np.float32)
    M, E = lg.shape
    b = _c(bias, np.float32)
    w = np.empty((M, K), np.float32)
    ids = np.empty((M, K), np.int32)
    src = np.empty((M, K), np.int32)
    rc = lib().oracle_topk(_p(lg), int(logits_bf16), M, E, K, SCORE[score], _p(b), int(renorm),
                           _p(w), _p(ids), _p(src))
    if rc != 0:
        raise ValueError("oracle_topk: invalid arguments")
    return w, ids, src


def permute(ids: np.ndarray, E: int):
    ids = _c(ids, np.int32)
    M, K = ids.shape
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(M * K, np.int32)
    inv = np.empty(M * K, np.int32)
    rc = lib().oracle_permute(_p(ids), M, K, E, _p(offsets), _p(perm), _p(inv))
    if rc != 0:
        raise ValueError("oracle_permute: expert id out of range")
    return offsets, perm, inv


def forward(shape, inp: dict, rows=None, routed_scale: float = 1.0):
    """Layer forward for token ``rows`` (default: all).  ``inp`` is a numpy input dict
    (see ``mixture_experts_layer_35_b200.inputs.to_numpy_inputs``); optional entries
    ``shared_gate`` ([H] BF16 bits: the shared expert's sigmoid gate row) and
    ``shared_out`` ([T,H] BF16 bits: a caller-computed shared output, used when there is
    no internal shared expert).  ``routed_scale`` multiplies the routed sum before its
    BF16 rounding.  Returns ``(out_bits[r,H], logits[r,E], w[r,K], ids[r,K])``."""
    x = _c(inp["x"], np.uint16)
    T, H = x.shape
    if rows is None:
        rows = np.arange(T, dtype=np.int32)
    rows = _c(rows, np.int32)
    keep = {}
    L = _Layer()
    L.T, L.H, L.I, L.E, L.K = T, shape.H, shape.I, shape.E, shape.K
    L.act, L.score, L.renorm = ACT[shape.act], SCORE[shape.score], int(shape.renorm)
    L.I_shared = shape.I_shared if inp.get("ws13") is not None else 0
    for name, dt in (("router_w", np.uint16), ("router_logits", np.float32), ("bias", np.float32),
                     ("w13", np.uint16), ("w2", np.uint16), ("ws13", np.uint16), ("ws2", np.uint16),
                     ("shared_gate", np.uint16), ("shared_out", np.uint16)):
        a = _c(inp.get(name), dt)
        keep[name] = a
        setattr(L, name, _p(a))
    L.routed_scale = float(routed_scale)
    n = len(rows)
    out = np.empty((n, H), np.uint16)
    lg = np.empty((n, shape.E), np.float32)
    w = np.empty((n, shape.K), np.float32)
    ids = np.empty((n, shape.K), np.int32)
    rc = lib().oracle_forward_rows(ctypes.byref(L), _p(x), _p(rows), n, _p(out), _p(lg), _p(w), _p(ids))
    if rc != 0:
        raise ValueError(f"oracle_forward_rows failed ({rc})")
    return out, lg, w, ids


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> float64 (exact widening)."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
