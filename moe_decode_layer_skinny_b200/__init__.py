"""Python binding of libkd.so, the B200 (sm_100a) MoE decode-layer library.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch is used for device memory and streams.  There is no CPU or
other fallback: if ``libkd.so`` is missing or fails to load, importing the
layer raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(HERE, "libkd.so")

KD_OK, KD_EINVAL, KD_ERANGE, KD_ECUDA, KD_ENOMEM, KD_ETIMEOUT, KD_EDEVICE = 0, -1, -2, -3, -4, -5, -6
KD_WBF16, KD_WFP8 = 0, 1
KD_STATIC_MAX_TOKENS, KD_STATIC_MAX_EXPERTS, KD_STATIC_MAX_HIDDEN = 64, 1024, 8192
T_H1F, T_H1B, T_LOGITS, T_IDX, T_GATES, T_COUNTS, T_NACTIVE, T_YSHARED, T_YROUTED, T_ATTN, \
    T_RESID, T_ACT, T_ACTSH = range(13)

# every symbol include/kd.h declares
EXPORTS = ("kd_layer_create", "kd_layer_destroy", "kd_decode_layer", "kd_decode_layer_full",
           "kd_layer_check",
           "kd_layer_qkv", "kd_layer_prefetch_l2", "kd_layer_debug_tensor", "kd_layer_read_weight",
           "kd_layer_bytes", "kd_layer_launches", "kd_layer_set_timing_events", "kd_stack_create",
           "kd_stack_run", "kd_stack_destroy", "kd_router_topk_static", "kd_last_error",
           "kd_tp_buffers", "kd_tp_attn", "kd_tp_router", "kd_tp_moe", "kd_tp_combine")
N_TIMING_EVENTS = 5


class KdError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"kd error {code}: {msg}")
        self.code = code


class _Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("q_heads", ctypes.c_int), ("kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("n_shared", ctypes.c_int), ("inter", ctypes.c_int), ("wdtype", ctypes.c_int),
                ("layer_id", ctypes.c_int), ("max_tokens", ctypes.c_int),
                ("router_bias", ctypes.c_void_p), ("mma_min_tokens", ctypes.c_int),
                ("full_layer", ctypes.c_int), ("rms_eps", ctypes.c_float),
                ("kv_n_seq", ctypes.c_int), ("kv_max_ctx", ctypes.c_int),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float),
                ("bias_select_only", ctypes.c_int), ("routed_scale", ctypes.c_float),
                ("tp_rank", ctypes.c_int), ("tp_size", ctypes.c_int),
                ("fp8_act_terms", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libkd.so (raises OSError if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(SO_PATH):
            raise OSError(f"{SO_PATH} is not built; run python -m moe_decode_layer_skinny_b200.build")
        L = ctypes.CDLL(SO_PATH)
        vp, i32, u64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
        L.kd_layer_create.argtypes = [ctypes.POINTER(_Config), u64, ctypes.POINTER(vp)]
        L.kd_layer_destroy.argtypes = [vp]
        L.kd_layer_destroy.restype = None
        L.kd_decode_layer.argtypes = [vp, vp, vp, i32, vp]
        L.kd_decode_layer_full.argtypes = [vp, vp, vp, vp, vp, vp, i32, vp]
        L.kd_layer_check.argtypes = [vp]
        L.kd_layer_qkv.argtypes = [vp]
        L.kd_layer_qkv.restype = vp
        L.kd_layer_prefetch_l2.argtypes = [vp, sz, vp]
        L.kd_layer_debug_tensor.argtypes = [vp, i32, ctypes.POINTER(vp)]
        L.kd_layer_read_weight.argtypes = [vp, i32, i32, i32, i32, vp, vp]
        L.kd_layer_bytes.argtypes = [vp, ctypes.POINTER(u64), ctypes.POINTER(u64)]
        L.kd_layer_launches.argtypes = [vp, ctypes.c_int]
        L.kd_layer_set_timing_events.argtypes = [vp, ctypes.POINTER(vp), i32]
        L.kd_stack_create.argtypes = [ctypes.POINTER(vp), i32, i32, i32, ctypes.POINTER(vp)]
        L.kd_stack_run.argtypes = [vp, vp, vp, vp]
        L.kd_stack_destroy.argtypes = [vp]
        L.kd_stack_destroy.restype = None
        L.kd_router_topk_static.argtypes = [vp, vp, i32, vp, vp, i32, i32, i32, i32, vp, vp, vp]
        L.kd_last_error.restype = ctypes.c_char_p
        fpp = ctypes.POINTER(vp)
        L.kd_tp_buffers.argtypes = [vp, fpp, fpp, fpp, fpp]
        L.kd_tp_attn.argtypes = [vp, vp, vp, i32, vp]
        L.kd_tp_router.argtypes = [vp, vp, i32, vp]
        L.kd_tp_moe.argtypes = [vp, i32, vp]
        L.kd_tp_combine.argtypes = [vp, vp, i32, vp]
        _lib = L
    return _lib


def _check(rc: int) -> None:
    if rc != KD_OK:
        raise KdError(rc, lib().kd_last_error().decode())


def _stream_ptr(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


@dataclass
class LayerSpec:
    hidden: int
    q_heads: int
    kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    n_shared: int
    inter: int
    wdtype: int = KD_WBF16
    layer_id: int = 0
    max_tokens: int = 64
    router_bias: np.ndarray | None = None
    mma_min_tokens: int = 0
    full_layer: int = 0
    rms_eps: float = 0.0
    kv_n_seq: int = 0
    kv_max_ctx: int = 0
    k_scale: float = 0.0
    v_scale: float = 0.0
    bias_select_only: int = 0
    routed_scale: float = 0.0
    tp_rank: int = 0
    tp_size: int = 0
    fp8_act_terms: int = 0

    @classmethod
    def from_dims(cls, dims, **kw) -> "LayerSpec":
        return cls(dims.hidden, dims.q_heads, dims.kv_heads, dims.head_dim, dims.n_experts,
                   dims.top_k, dims.n_shared, dims.inter, **kw)


class Layer:
    """One decode layer on the current CUDA device (kd_layer_*)."""

    def __init__(self, spec: LayerSpec, seed: int = 0):
        self.spec = spec
        bias = None
        if spec.router_bias is not None:
            bias = np.ascontiguousarray(spec.router_bias, np.float32)
        cfg = _Config(spec.hidden, spec.q_heads, spec.kv_heads, spec.head_dim, spec.n_experts,
                      spec.top_k, spec.n_shared, spec.inter, spec.wdtype, spec.layer_id,
                      spec.max_tokens, None if bias is None else bias.ctypes.data,
                      spec.mma_min_tokens, spec.full_layer, spec.rms_eps, spec.kv_n_seq,
                      spec.kv_max_ctx, spec.k_scale, spec.v_scale, spec.bias_select_only,
                      spec.routed_scale, spec.tp_rank, spec.tp_size, spec.fp8_act_terms)
        h = ctypes.c_void_p()
        _check(lib().kd_layer_create(ctypes.byref(cfg), seed, ctypes.byref(h)))
        self._h = h

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def close(self) -> None:
        if self._h:
            lib().kd_layer_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def decode(self, hidden, attn_out, M: int | None = None, stream=None) -> None:
        """kd_decode_layer on torch CUDA tensors (bf16, contiguous): hidden [M,H]
        is updated in place."""
        if M is None:
            M = hidden.shape[0]
        _check(lib().kd_decode_layer(self._h, hidden.data_ptr(), attn_out.data_ptr(), M,
                                     _stream_ptr(stream)))

    def decode_full(self, hidden, k_cache, v_cache, seq, pos, M: int | None = None,
                    stream=None) -> None:
        """kd_decode_layer_full on torch CUDA tensors: hidden bf16 [M,H] (in
        place), k_cache / v_cache uint8 e4m3 codes [n_seq, max_ctx, kv_heads *
        head_dim] (the M new positions are written), seq / pos int32 [M]."""
        if M is None:
            M = hidden.shape[0]
        _check(lib().kd_decode_layer_full(self._h, hidden.data_ptr(), k_cache.data_ptr(),
                                          v_cache.data_ptr(), seq.data_ptr(), pos.data_ptr(), M,
                                          _stream_ptr(stream)))

    # ---- tensor-parallel shard (spec.tp_size > 1): the four phases of
    # kd_tp_*; the exchanges between them are the caller's (tp.decode_tp)
    def tp_buffers(self) -> dict:
        """Device pointers of the shard's fp32 exchange buffers (kd_tp_buffers)."""
        ptrs = [ctypes.c_void_p() for _ in range(4)]
        _check(lib().kd_tp_buffers(self._h, *[ctypes.byref(p) for p in ptrs]))
        return dict(zip(("p", "lshard", "lfull", "y"), (p.value for p in ptrs)))

    def tp_attn(self, hidden, attn, M: int | None = None, stream=None) -> None:
        M = hidden.shape[0] if M is None else M
        _check(lib().kd_tp_attn(self._h, hidden.data_ptr(), attn.data_ptr(), M, _stream_ptr(stream)))

    def tp_router(self, hidden, M: int | None = None, stream=None) -> None:
        M = hidden.shape[0] if M is None else M
        _check(lib().kd_tp_router(self._h, hidden.data_ptr(), M, _stream_ptr(stream)))

    def tp_moe(self, M: int, stream=None) -> None:
        _check(lib().kd_tp_moe(self._h, M, _stream_ptr(stream)))

    def tp_combine(self, hidden, M: int | None = None, stream=None) -> None:
        M = hidden.shape[0] if M is None else M
        _check(lib().kd_tp_combine(self._h, hidden.data_ptr(), M, _stream_ptr(stream)))

    def decode_ptr(self, hidden_ptr: int, attn_ptr: int, M: int, stream_ptr: int | None) -> int:
        return lib().kd_decode_layer(self._h, hidden_ptr, attn_ptr, M, stream_ptr)

    def check(self) -> None:
        _check(lib().kd_layer_check(self._h))

    def qkv_ptr(self) -> int:
        return lib().kd_layer_qkv(self._h)

    def debug_ptr(self, which: int) -> int:
        p = ctypes.c_void_p()
        _check(lib().kd_layer_debug_tensor(self._h, which, ctypes.byref(p)))
        return p.value

    def prefetch_l2(self, max_bytes: int = 0, stream=None) -> None:
        _check(lib().kd_layer_prefetch_l2(self._h, max_bytes, _stream_ptr(stream)))

    def set_timing_events(self, events) -> None:
        """torch.cuda.Event list (enable_timing=True) of length N_TIMING_EVENTS, or None."""
        if not events:
            _check(lib().kd_layer_set_timing_events(self._h, None, 0))
            return
        if any(not e.cuda_event for e in events):
            raise ValueError("timing events must have been recorded once (torch creates them lazily)")
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        _check(lib().kd_layer_set_timing_events(self._h, arr, len(events)))

    def launches(self, M: int) -> int:
        """Kernels one decode call with M tokens launches."""
        n = lib().kd_layer_launches(self._h, M)
        if n < 0:
            _check(n)
        return n

    def bytes(self) -> tuple[int, int]:
        a, b = ctypes.c_uint64(), ctypes.c_uint64()
        _check(lib().kd_layer_bytes(self._h, ctypes.byref(a), ctypes.byref(b)))
        return a.value, b.value

    def read_weight(self, kind: int, expert: int, row0: int, nrows: int):
        """Logical rows of one weight matrix: bf16 bits (uint16) or (e4m3 codes,
        scales of the covered 128-row blocks)."""
        s = self.spec
        K = {1: s.hidden, 2: s.q_heads * s.head_dim, 3: s.hidden, 4: s.hidden, 5: s.hidden,
             6: s.inter}[kind]
        if s.wdtype == KD_WBF16:
            out = np.empty((nrows, K), np.uint16)
            _check(lib().kd_layer_read_weight(self._h, kind, expert, row0, nrows, out.ctypes.data, None))
            return out
        out = np.empty((nrows, K), np.uint8)
        nb = (row0 + nrows - 1) // 128 - row0 // 128 + 1
        sc = np.empty((nb, (K + 127) // 128), np.float32)
        _check(lib().kd_layer_read_weight(self._h, kind, expert, row0, nrows, out.ctypes.data,
                                          sc.ctypes.data))
        return out, sc


def router_topk_static(router_w, router_scales, wdtype: int, router_bias, h1, M: int,
                       hidden: int, n_experts: int, top_k: int, idx_out, gates_out,
                       stream=None) -> None:
    """kd_router_topk_static on torch CUDA tensors (or None for the optional
    ones); allocates no device memory.  The tensors are checked here (device,
    contiguity, dtype, size) so that a wrong one raises instead of being read
    or written out of bounds by the kernel."""
    import torch

    def need(t, name, dtypes, numel):
        if t is None:
            raise ValueError(f"router_topk_static: {name} is required")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"router_topk_static: {name} must be a contiguous CUDA tensor")
        if t.dtype not in dtypes:
            raise ValueError(f"router_topk_static: {name} has dtype {t.dtype}, want {dtypes}")
        if t.numel() < numel:
            raise ValueError(f"router_topk_static: {name} has {t.numel()} elements, needs {numel}")

    if M >= 1 and n_experts >= 1 and top_k >= 1 and hidden >= 1:
        wt = (torch.bfloat16, torch.int16, torch.uint16) if wdtype == KD_WBF16 else \
            (torch.uint8, torch.float8_e4m3fn)
        need(router_w, "router_w", wt, n_experts * hidden)
        if wdtype == KD_WFP8:
            need(router_scales, "router_scales", (torch.float32,),
                 ((n_experts + 127) // 128) * ((hidden + 127) // 128))
        if router_bias is not None:
            need(router_bias, "router_bias", (torch.float32,), n_experts)
        need(h1, "h1", (torch.float32,), M * hidden)
        need(idx_out, "idx_out", (torch.int32,), M * top_k)
        need(gates_out, "gates_out", (torch.float32,), M * top_k)
    ptr = lambda t: None if t is None else t.data_ptr()
    _check(lib().kd_router_topk_static(ptr(router_w), ptr(router_scales), wdtype, ptr(router_bias),
                                       ptr(h1), M, hidden, n_experts, top_k, ptr(idx_out),
                                       ptr(gates_out), _stream_ptr(stream)))


class Stack:
    """Multi-layer decode step captured in a CUDA graph (kd_stack_*)."""

    def __init__(self, layers: list[Layer], M: int, prefetch: bool = True):
        arr = (ctypes.c_void_p * len(layers))(*[l.handle.value for l in layers])
        h = ctypes.c_void_p()
        _check(lib().kd_stack_create(arr, len(layers), M, 1 if prefetch else 0, ctypes.byref(h)))
        self._h = h
        self._layers = layers

    def run(self, hidden, attn_out, stream=None) -> None:
        _check(lib().kd_stack_run(self._h, hidden.data_ptr(), attn_out.data_ptr(), _stream_ptr(stream)))

    def close(self) -> None:
        if self._h:
            lib().kd_stack_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
