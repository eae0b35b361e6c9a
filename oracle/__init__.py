"""CPU oracle of the MoE decode layer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The product (the CUDA library and its
binding) never calls it and there is no CPU fallback anywhere.

``liboracle.so`` is a plain single-pass fp64 C implementation of the layer
(see ``orc.h`` for the equations and the pages they follow).  It shares no code
with the CUDA path; the only common module is the seeded input generator
``kdgen``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = [os.path.join(_HERE, "orc.c"), os.path.join(_HERE, "orc.h"),
        os.path.join(_HERE, "..", "kdgen", "kd_gen.h")]


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (fp64, no fast-math, no FMA contraction)."""
    stale = not os.path.exists(_SO) or any(os.path.getmtime(s) > os.path.getmtime(_SO) for s in _SRC)
    if force or stale:
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                               "-o", _SO, _SRC[0], "-lm"])
    return _SO


class _Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("q_heads", ctypes.c_int), ("kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("n_shared", ctypes.c_int), ("inter", ctypes.c_int), ("wdtype", ctypes.c_int),
                ("layer_id", ctypes.c_int), ("seed", ctypes.c_uint64)]


class _W(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("wqkv", "wo", "wr", "wg", "wu", "wd")]


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        vp = ctypes.c_void_p
        L.orc_layer.restype = ctypes.c_int
        L.orc_layer.argtypes = [ctypes.POINTER(_Cfg), ctypes.POINTER(_W), vp, vp, vp, ctypes.c_int,
                                vp, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp, vp]
        L.orc_weight_rows.restype = ctypes.c_int
        L.orc_weight_rows.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, vp]
        L.orc_bf16_value.restype = ctypes.c_double
        L.orc_bf16_value.argtypes = [ctypes.c_uint16]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        _lib = L
    return _lib


def _cfg(dims, wdtype=0, layer_id=0, seed=0) -> _Cfg:
    return _Cfg(dims.hidden, dims.q_heads, dims.kv_heads, dims.head_dim, dims.n_experts,
                dims.top_k, dims.n_shared, dims.inter, wdtype, layer_id, seed)


def _p(a):
    if a is None:
        return None
    assert a.flags.c_contiguous
    return a.ctypes.data


def bf16_value(bits: int) -> float:
    return lib().orc_bf16_value(bits)


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(code)


def weight_rows(dims, kind: int, expert: int, row0: int, nrows: int, wdtype=0, layer_id=0,
                seed=0) -> np.ndarray:
    """Decoded logical rows of one generated weight matrix (fp64)."""
    c = _cfg(dims, wdtype, layer_id, seed)
    K = {1: dims.hidden, 2: dims.attn, 3: dims.hidden, 4: dims.hidden, 5: dims.hidden,
         6: dims.inter}[kind]
    out = np.empty((nrows, K), np.float64)
    rc = lib().orc_weight_rows(ctypes.byref(c), kind, expert, row0, nrows, _p(out))
    if rc != 0:
        raise ValueError("orc_weight_rows: bad arguments")
    return out


def layer(dims, x, attn, *, wdtype=0, layer_id=0, seed=0, bias=None, weights=None,
          forced_idx=None, ksplit=1, nthreads=None, want_qkv=True) -> dict:
    """Evaluate one layer for M tokens.

    x, attn: fp64 arrays [M, H], [M, A] (the exact values the GPU receives,
    e.g. decoded bf16).  weights: optional dict of explicit fp64 logical
    weights (wqkv, wo, wr, wg, wu, wd; expert arrays shared-first).
    Returns fp64 qkv, h1, logits, gates, out and int32 idx.
    """
    x = np.ascontiguousarray(x, np.float64)
    attn = np.ascontiguousarray(attn, np.float64)
    M = x.shape[0]
    assert x.shape == (M, dims.hidden) and attn.shape == (M, dims.attn)
    c = _cfg(dims, wdtype, layer_id, seed)
    keep = []
    wp = None
    if weights is not None:
        arrs = {k: np.ascontiguousarray(weights[k], np.float64) for k in ("wqkv", "wo", "wr", "wg", "wu", "wd")}
        keep.append(arrs)
        wp = ctypes.byref(_W(*(arrs[k].ctypes.data for k in ("wqkv", "wo", "wr", "wg", "wu", "wd"))))
    b = None if bias is None else np.ascontiguousarray(bias, np.float64)
    f = None if forced_idx is None else np.ascontiguousarray(forced_idx, np.int32)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    res = {
        "qkv": np.zeros((M, dims.nqkv)) if want_qkv else None,
        "h1": np.zeros((M, dims.hidden)),
        "logits": np.zeros((M, dims.n_experts)),
        "idx": np.zeros((M, dims.top_k), np.int32),
        "gates": np.zeros((M, dims.top_k)),
        "out": np.zeros((M, dims.hidden)),
    }
    rc = lib().orc_layer(ctypes.byref(c), wp, _p(b), _p(x), _p(attn), M, _p(f), ksplit, nthreads,
                         _p(res["qkv"]), _p(res["h1"]), _p(res["logits"]), _p(res["idx"]),
                         _p(res["gates"]), _p(res["out"]))
    if rc != 0:
        raise ValueError("orc_layer: bad arguments")
    return res
