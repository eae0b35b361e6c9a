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
                ("layer_id", ctypes.c_int), ("seed", ctypes.c_uint64),
                ("bias_select_only", ctypes.c_int), ("routed_scale", ctypes.c_double)]


_WNAMES = ("wqkv", "wo", "wr", "wg", "wu", "wd", "g1", "g2")


class _W(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _WNAMES]


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
        L.orc_e4m3_code.restype = ctypes.c_uint8
        L.orc_e4m3_code.argtypes = [ctypes.c_double]
        L.orc_rmsnorm.restype = None
        L.orc_rmsnorm.argtypes = [vp, vp, ctypes.c_int, ctypes.c_double, vp]
        i32, f64 = ctypes.c_int, ctypes.c_double
        L.orc_attention.restype = i32
        L.orc_attention.argtypes = [vp, i32, vp, vp, f64, f64, i32, i32, i32, i32, i32, vp, vp, i32,
                                    vp, i32]
        L.orc_layer_full.restype = i32
        L.orc_layer_full.argtypes = [ctypes.POINTER(_Cfg), ctypes.POINTER(_W), vp, vp, i32, vp, vp,
                                     f64, f64, i32, i32, vp, vp, f64, i32, vp, i32,
                                     vp, vp, vp, vp, vp, vp, vp, vp]
        _lib = L
    return _lib


def _cfg(dims, wdtype=0, layer_id=0, seed=0, bias_select_only=False, routed_scale=1.0) -> _Cfg:
    return _Cfg(dims.hidden, dims.q_heads, dims.kv_heads, dims.head_dim, dims.n_experts,
                dims.top_k, dims.n_shared, dims.inter, wdtype, layer_id, seed,
                1 if bias_select_only else 0, routed_scale)


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


def _weights_ptr(weights, keep):
    if weights is None:
        return None
    arrs = {k: np.ascontiguousarray(weights[k], np.float64) for k in _WNAMES if k in weights}
    keep.append(arrs)
    return ctypes.byref(_W(*(arrs[k].ctypes.data if k in arrs else None for k in _WNAMES)))


def e4m3_code(v: float) -> int:
    return int(lib().orc_e4m3_code(float(v)))


def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    """RMSNorm of each row of x [.., n] with gain gamma [n]."""
    x = np.ascontiguousarray(x, np.float64)
    g = np.ascontiguousarray(gamma, np.float64)
    flat = x.reshape(-1, x.shape[-1])
    out = np.empty_like(flat)
    for i in range(flat.shape[0]):
        lib().orc_rmsnorm(_p(flat[i]), _p(g), flat.shape[1], eps, _p(out[i]))
    return out.reshape(x.shape)


def attention(q, kc, vc, k_scale, v_scale, hq, hkv, hd, seq, pos) -> np.ndarray:
    """Attention of rows q [M, hq*hd] over e4m3 caches kc, vc [n_seq, max_ctx, hkv*hd]."""
    q = np.ascontiguousarray(q, np.float64)
    kc = np.ascontiguousarray(kc, np.uint8)
    vc = np.ascontiguousarray(vc, np.uint8)
    seq = np.ascontiguousarray(seq, np.int32)
    pos = np.ascontiguousarray(pos, np.int32)
    M = q.shape[0]
    out = np.zeros((M, hq * hd))
    rc = lib().orc_attention(_p(q), q.shape[1], _p(kc), _p(vc), k_scale, v_scale, kc.shape[0],
                             kc.shape[1], hq, hkv, hd, _p(seq), _p(pos), M, _p(out), hq * hd)
    if rc != 0:
        raise ValueError("orc_attention: bad arguments")
    return out


def layer_full(dims, x, kc, vc, k_scale, v_scale, seq, pos, *, wdtype=0, layer_id=0, seed=0,
               eps=1e-6, bias=None, weights=None, keep_new_kv=False, forced_idx=None,
               nthreads=None) -> dict:
    """The full decode layer (RMSNorm, QKV, FP8-cache attention, o-proj +
    residual, RMSNorm, MoE) for M tokens; kc / vc [n_seq, max_ctx, kv_heads*hd]
    e4m3 codes are copied, and the copies (with the new tokens' codes) are
    returned as "kc" / "vc"."""
    x = np.ascontiguousarray(x, np.float64)
    M = x.shape[0]
    kc = np.array(kc, np.uint8, copy=True, order="C")
    vc = np.array(vc, np.uint8, copy=True, order="C")
    seq = np.ascontiguousarray(seq, np.int32)
    pos = np.ascontiguousarray(pos, np.int32)
    c = _cfg(dims, wdtype, layer_id, seed)
    keep = []
    wp = _weights_ptr(weights, keep)
    b = None if bias is None else np.ascontiguousarray(bias, np.float64)
    f = None if forced_idx is None else np.ascontiguousarray(forced_idx, np.int32)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    res = {"qkv": np.zeros((M, dims.nqkv)), "attn": np.zeros((M, dims.attn)),
           "h1": np.zeros((M, dims.hidden)), "v": np.zeros((M, dims.hidden)),
           "logits": np.zeros((M, dims.n_experts)), "idx": np.zeros((M, dims.top_k), np.int32),
           "gates": np.zeros((M, dims.top_k)), "out": np.zeros((M, dims.hidden))}
    rc = lib().orc_layer_full(ctypes.byref(c), wp, _p(b), _p(x), M, _p(kc), _p(vc), k_scale,
                              v_scale, kc.shape[0], kc.shape[1], _p(seq), _p(pos), eps,
                              1 if keep_new_kv else 0, _p(f), nthreads, _p(res["qkv"]),
                              _p(res["attn"]), _p(res["h1"]), _p(res["v"]), _p(res["logits"]),
                              _p(res["idx"]), _p(res["gates"]), _p(res["out"]))
    if rc != 0:
        raise ValueError("orc_layer_full: bad arguments")
    res["kc"], res["vc"] = kc, vc
    return res


def layer(dims, x, attn, *, wdtype=0, layer_id=0, seed=0, bias=None, weights=None,
          forced_idx=None, ksplit=1, nthreads=None, want_qkv=True, bias_select_only=False,
          routed_scale=1.0) -> dict:
    """Evaluate one layer for M tokens.

    x, attn: fp64 arrays [M, H], [M, A] (the exact values the GPU receives,
    e.g. decoded bf16).  weights: optional dict of explicit fp64 logical
    weights (wqkv, wo, wr, wg, wu, wd; expert arrays shared-first).
    Returns fp64 qkv, h1, logits, gates, out and int32 idx.  bias_select_only:
    the bias chooses the experts only (gates from the unbiased logits, which
    are then the returned logits); routed_scale: factor on the routed sum.
    """
    x = np.ascontiguousarray(x, np.float64)
    attn = np.ascontiguousarray(attn, np.float64)
    M = x.shape[0]
    assert x.shape == (M, dims.hidden) and attn.shape == (M, dims.attn)
    c = _cfg(dims, wdtype, layer_id, seed, bias_select_only, routed_scale)
    keep = []
    wp = _weights_ptr(weights, keep)
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
