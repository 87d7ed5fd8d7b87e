"""CPU oracle of the latent-MoE decode block (fp64, plain C).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product package never
imports this module, and this module imports nothing from the product.

``moe_oracle.c`` holds the arithmetic; this file only compiles it (``gcc``),
loads it with ctypes and marshals numpy arrays in and out.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                               "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("latent", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("expert_inter", ctypes.c_int32), ("shared_inter", ctypes.c_int32),
                ("score_fn", ctypes.c_int32), ("renormalize", ctypes.c_int32),
                ("routed_scale", ctypes.c_double)]


_P = ctypes.c_void_p


class _Weights(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("router_w", "router_bias", "w_in", "w_out", "gu_codes",
                                  "gu_scales", "dn_codes", "dn_scales", "sh_gate", "sh_up",
                                  "sh_down")]


class _Outputs(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("logits", "keys", "ids", "weights", "margin", "z", "h", "y",
                                  "c", "h_s", "o_s", "out")]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_forward.argtypes = [ctypes.POINTER(_Cfg), ctypes.POINTER(_Weights), _P,
                                       ctypes.c_int32, ctypes.POINTER(_Outputs)]
        lib.oracle_forward.restype = ctypes.c_int
        lib.oracle_route.argtypes = [ctypes.POINTER(_Cfg), ctypes.POINTER(_Weights), _P,
                                     ctypes.c_int32, _P, _P, _P, _P, _P]
        lib.oracle_route.restype = ctypes.c_int
        lib.oracle_dequant_mx.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int64, _P]
        lib.oracle_dequant_mx.restype = None
        lib.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_value.restype = ctypes.c_double
        lib.oracle_e8m0_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e8m0_value.restype = ctypes.c_double
        lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_value.restype = ctypes.c_double
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = None
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_P)


def _cfg(shape) -> _Cfg:
    return _Cfg(shape.hidden, shape.latent, shape.num_experts, shape.top_k, shape.expert_inter,
                shape.shared_inter, shape.score_fn, shape.renormalize, float(shape.routed_scale))


def _weights(w: dict):
    keep = {}
    for k, v in w.items():
        if v is not None:
            keep[k] = np.ascontiguousarray(v)
    ws = _Weights(**{f[0]: _ptr(keep.get(f[0])) for f in _Weights._fields_})
    return ws, keep


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_threads(n: int) -> None:
    """Threads of the oracle's token loop (for timing; results do not change)."""
    _load().oracle_set_threads(int(n))


def e2m1_value(code: int) -> float:
    return float(_load().oracle_e2m1_value(code))


def e8m0_value(s: int) -> float:
    return float(_load().oracle_e8m0_value(s))


def bf16_value(bits: int) -> float:
    return float(_load().oracle_bf16_value(bits))


def dequant_mx(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """[rows][K/2] codes + [rows][K/32] e8m0 scales -> float64 [rows][K]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, half = codes.shape
    K = half * 2
    assert scales.shape == (rows, K // 32)
    out = np.empty((rows, K), dtype=np.float64)
    _load().oracle_dequant_mx(_ptr(codes), _ptr(scales), rows, K, _ptr(out))
    return out


def forward(shape, w: dict, x: np.ndarray, intermediates: bool = True) -> dict:
    """Run the whole block on B tokens; returns float64 arrays (ids int32)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B = x.shape[0]
    H, L, E, k, I, Is = (shape.hidden, shape.latent, shape.num_experts, shape.top_k,
                         shape.expert_inter, shape.shared_inter)
    assert x.shape == (B, H)
    r = {"out": np.zeros((B, H)), "ids": np.zeros((B, k), np.int32), "weights": np.zeros((B, k)),
         "margin": np.zeros(B), "logits": np.zeros((B, E)), "keys": np.zeros((B, E))}
    if intermediates:
        r.update(z=np.zeros((B, L)), h=np.zeros((B, k, I)), y=np.zeros((B, k, L)),
                 c=np.zeros((B, L)), h_s=np.zeros((B, max(Is, 1))), o_s=np.zeros((B, H)))
    o = _Outputs(**{n: _ptr(r.get(n)) for n in [f[0] for f in _Outputs._fields_]})
    ws, keep = _weights(w)
    rc = lib.oracle_forward(ctypes.byref(_cfg(shape)), ctypes.byref(ws), _ptr(x), B, ctypes.byref(o))
    if rc != 0:
        raise ValueError("oracle_forward rejected its arguments (code %d)" % rc)
    del keep
    return r


def route(shape, w: dict, x: np.ndarray) -> dict:
    """Router, scores and top-k only."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B = x.shape[0]
    E, k = shape.num_experts, shape.top_k
    r = {"logits": np.zeros((B, E)), "keys": np.zeros((B, E)), "ids": np.zeros((B, k), np.int32),
         "weights": np.zeros((B, k)), "margin": np.zeros(B)}
    ws, keep = _weights(w)
    rc = lib.oracle_route(ctypes.byref(_cfg(shape)), ctypes.byref(ws), _ptr(x), B,
                          _ptr(r["logits"]), _ptr(r["keys"]), _ptr(r["ids"]), _ptr(r["weights"]),
                          _ptr(r["margin"]))
    if rc != 0:
        raise ValueError("oracle_route rejected its arguments (code %d)" % rc)
    del keep
    return r
