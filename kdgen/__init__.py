"""Seeded, counter-based synthetic inputs for the MoE decode layer.

Shared by the CUDA library's tests and benchmark and by the CPU oracle's
tests: it only produces inputs (activations, router bias, reference copies of
generated weights) and holds none of the layer's arithmetic.  The definition
of the generator is in ``kd_gen.h``; this module calls the same C code through
``libkdgen.so``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libkdgen.so")
_SRC = [os.path.join(_HERE, "kdgen_host.c"), os.path.join(_HERE, "kd_gen.h")]

# tensor kinds of kd_gen.h
QKV, OPROJ, ROUTER, GATE, UP, DOWN, HIDDEN_IN, ATTN_OUT = 1, 2, 3, 4, 5, 6, 16, 17
NORM1, NORM2, KCACHE, VCACHE = 7, 8, 18, 19
UNIT = float.fromhex("0x1.bb67aep-16")
W002 = float.fromhex("0x1.1bc77ap-21")


def build(force: bool = False) -> str:
    """Compile libkdgen.so with gcc (no fast-math, no FMA contraction)."""
    stale = not os.path.exists(_SO) or any(os.path.getmtime(s) > os.path.getmtime(_SO) for s in _SRC)
    if force or stale:
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", _SO,
                               _SRC[0], "-lm"])
    return _SO


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        u64, i64, u32, f32, f64, i32 = (ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint32,
                                        ctypes.c_float, ctypes.c_double, ctypes.c_int)
        vp = ctypes.c_void_p
        L.kdg_host_mix.restype = u64; L.kdg_host_mix.argtypes = [u64]
        L.kdg_host_stream.restype = u64; L.kdg_host_stream.argtypes = [u64, u64]
        L.kdg_host_uid.restype = u64; L.kdg_host_uid.argtypes = [u32, u32, u32]
        L.kdg_host_ih4.restype = i32; L.kdg_host_ih4.argtypes = [u64]
        L.kdg_host_values.argtypes = [u64, u64, u64, i64, f32, vp]
        L.kdg_host_bf16.argtypes = [vp, i64, vp]
        L.kdg_host_e4m3.argtypes = [vp, i64, vp]
        L.kdg_host_activations.argtypes = [u64, u32, u32, i32, i32, f64, vp]
        L.kdg_host_zipf_bias.argtypes = [i32, f64, vp]
        L.kdg_host_weight_bf16.argtypes = [u64, u32, u32, u32, i32, i32, vp]
        L.kdg_host_weight_fp8.argtypes = [u64, u32, u32, u32, i32, i32, vp, vp]
        L.kdg_host_norm_bf16.argtypes = [u64, u32, u32, i32, vp]
        L.kdg_host_kv_cache.argtypes = [u64, u32, u32, i32, i32, i32, f32, f32, vp]
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags.c_contiguous
    return a.ctypes.data


def mix(z: int) -> int:
    return lib().kdg_host_mix(z)


def uid(layer: int, kind: int, slot: int = 0) -> int:
    return lib().kdg_host_uid(layer, kind, slot)


def values(seed: int, tensor_uid: int, start: int, n: int, c: float = UNIT) -> np.ndarray:
    out = np.empty(n, np.float32)
    lib().kdg_host_values(seed, tensor_uid, start, n, c, _p(out))
    return out


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().kdg_host_bf16(_p(x), x.size, _p(out))
    return out


def to_e4m3_codes(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().kdg_host_e4m3(_p(x), x.size, _p(out))
    return out


def activations(seed: int, layer: int, kind: int, M: int, width: int, rho: float = 0.0) -> np.ndarray:
    """bf16 bits [M, width]; rows follow x_t = rho x_{t-1} + sqrt(1-rho^2) z_t."""
    out = np.empty((M, width), np.uint16)
    lib().kdg_host_activations(seed, layer, kind, M, width, rho, _p(out))
    return out


def zipf_bias(E: int, s: float) -> np.ndarray:
    out = np.empty(E, np.float32)
    lib().kdg_host_zipf_bias(E, s, _p(out))
    return out


def weight_bf16(seed: int, layer: int, kind: int, slot: int, R: int, K: int) -> np.ndarray:
    out = np.empty((R, K), np.uint16)
    lib().kdg_host_weight_bf16(seed, layer, kind, slot, R, K, _p(out))
    return out


def weight_fp8(seed: int, layer: int, kind: int, slot: int, R: int, K: int):
    codes = np.empty((R, K), np.uint8)
    scales = np.empty(((R + 127) // 128, (K + 127) // 128), np.float32)
    lib().kdg_host_weight_fp8(seed, layer, kind, slot, R, K, _p(codes), _p(scales))
    return codes, scales


def norm_bf16(seed: int, layer: int, kind: int, n: int) -> np.ndarray:
    """RMSNorm gains [n] (kind NORM1 / NORM2) as bf16 bits."""
    out = np.empty(n, np.uint16)
    lib().kdg_host_norm_bf16(seed, layer, kind, n, _p(out))
    return out


def kv_cache(seed: int, layer: int, kind: int, n_seq: int, max_ctx: int, width: int,
             sigma: float, scale: float) -> np.ndarray:
    """Synthetic e4m3 KV-cache codes [n_seq, max_ctx, width] (kind KCACHE / VCACHE)."""
    out = np.empty((n_seq, max_ctx, width), np.uint8)
    lib().kdg_host_kv_cache(seed, layer, kind, n_seq, max_ctx, width, sigma, scale, _p(out))
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------- workloads

@dataclass(frozen=True)
class Dims:
    hidden: int
    q_heads: int
    kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    n_shared: int
    inter: int

    @property
    def nqkv(self) -> int:
        return (self.q_heads + 2 * self.kv_heads) * self.head_dim

    @property
    def attn(self) -> int:
        return self.q_heads * self.head_dim


TINY = Dims(hidden=256, q_heads=4, kv_heads=1, head_dim=64, n_experts=8, top_k=2, n_shared=1, inter=128)
K2 = Dims(hidden=7168, q_heads=64, kv_heads=8, head_dim=128, n_experts=256, top_k=8, n_shared=1, inter=2048)


@dataclass(frozen=True)
class Workload:
    name: str
    dims: Dims
    M: int
    wdtype: int = 0            # 0 bf16, 1 FP8 e4m3 with 128x128 fp32 block scales
    rho: float = 0.0           # token-axis correlation of the activations
    zipf_s: float = 0.0        # > 0: router bias -s ln(e+1) added before the top-k
    n_layers: int = 1
    seed: int = 0
    desc: str = field(default="", compare=False)

    def bias(self):
        return zipf_bias(self.dims.n_experts, self.zipf_s) if self.zipf_s > 0 else None

    def hidden_in(self) -> np.ndarray:
        return activations(self.seed, 0, HIDDEN_IN, self.M, self.dims.hidden, self.rho)

    def attn_out(self, layer: int = 0) -> np.ndarray:
        return activations(self.seed, layer, ATTN_OUT, self.M, self.dims.attn, self.rho)


WORKLOADS = {
    "tiny": Workload("tiny", TINY, 1, desc="tiny layer, M=1, bf16"),
    "batch1": Workload("batch1", K2, 1, desc="H=7168 layer, M=1, bf16, uniform routing"),
    "verify8": Workload("verify8", K2, 8, rho=0.9,
                        desc="H=7168 layer, M=8 speculative-verify rows with 0.9 correlation, bf16"),
    "batch64_zipf": Workload("batch64_zipf", K2, 64, zipf_s=1.1,
                             desc="H=7168 layer, M=64, Zipf(1.1) router bias, bf16"),
    "stack4_fp8": Workload("stack4_fp8", K2, 32, wdtype=1, n_layers=4,
                           desc="4 H=7168 layers, M=32, FP8 e4m3 128x128-block weights"),
}
