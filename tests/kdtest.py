"""Helpers shared by the GPU parity tests: run the CUDA layer through the C ABI
and compare it with the CPU oracle.

Tolerances (from the layer's precision contract): per output tensor,
max|gpu - oracle| / rms(oracle) <= 1e-2 for bf16 weights, 3e-2 for FP8.
Both outputs (the layer output and qkv) are bf16 by the interface, and the
correctly rounded bf16 value of the exact result is itself up to half a bf16
ulp away from it -- up to 2^-9 max|x|, which exceeds 1e-2 rms wherever
max|x| > 5.1 rms.  So each comparison asserts three things:
  * raw    max|gpu - oracle| / rms <= tol + max half-ulp(oracle) / rms (the
           bound every correctly rounded result meets), and the literal bound
           max|gpu - oracle| / rms <= tol wherever bf16 storage leaves room for
           it (max half-ulp(oracle) / rms <= tol);
  * excess the error beyond that storage rounding (rel_err_bf16) <= tol;
  * tight  the excess <= TIGHT[wdtype], a bound set from the arithmetic of the
           kernels (bf16 weights: exact products of hi + lo activation terms,
           fp32 accumulation; measured ~5e-5), low enough that dropping an
           activation term (~1e-2) fails.
The top-k expert ids must match exactly unless the oracle's k-th and
(k+1)-th logits are closer than 1e-4, in which case that token's row is
compared with the oracle recomputed under the GPU's selection.
"""
from __future__ import annotations

import numpy as np

import kdgen
import oracle

# key 2: FP8 weights with one e4m3 term per expert activation (W8A8): each
# activation carries one e4m3 rounding (relative <= 2^-4, rms 2^-4 / sqrt(3)
# for a uniform rounding error) at each of the two expert matrices, so the
# output's error is bounded in rms, not elementwise: rms(gpu - oracle) <= 2^-4
# rms(oracle) (sqrt(2) x 2^-4 / sqrt(3) ~ 0.051 for two independent stages),
# and its largest element within 8 such rms (a sanity bound).
TOL = {0: 1e-2, 1: 3e-2, 2: 2.0 ** -4}
TIGHT = {0: 1e-3, 1: 3e-2, 2: 2.0 ** -4}
TIE_GAP = 1e-4


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return kdgen.bf16_bits_to_f32(bits).astype(np.float64)


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    """max|gpu - ref| / rms(ref)."""
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
    return float(np.max(np.abs(gpu.astype(np.float64) - ref))) / max(rms, 1e-300)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Largest error of round-to-nearest into bf16 (8 significant bits) at x."""
    ax = np.abs(x.astype(np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def rel_err_bf16(gpu: np.ndarray, ref: np.ndarray) -> float:
    """max over elements of (|gpu - ref| - half-ulp_bf16(ref))+ / rms(ref).

    A bf16 result cannot be closer to the exact value than the rounding of
    that value into bf16; this measures the error beyond that storage
    rounding (which alone is ~1% of rms where max|x| ~ 4 rms)."""
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
    ex = np.abs(gpu.astype(np.float64) - ref) - bf16_half_ulp(ref)
    return float(max(np.max(ex), 0.0)) / max(rms, 1e-300)


def rounding_floor(ref: np.ndarray) -> float:
    """max half-ulp_bf16(ref) / rms(ref): what bf16 storage of the exact value
    alone may cost."""
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
    return float(np.max(bf16_half_ulp(ref))) / max(rms, 1e-300)


def check_output(report: dict, key: str, gpu: np.ndarray, ref: np.ndarray, wdtype: int,
                 strict_raw=None) -> None:
    """Raw, beyond-rounding and tight checks of one bf16 output tensor.
    strict_raw: assert the literal raw bound (None: wherever the correctly
    rounded result meets it)."""
    tol = TOL[wdtype]
    if wdtype == 2:   # W8A8: the rms bound (see TOL)
        err = gpu.astype(np.float64) - ref
        rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
        report[key + "_rms"] = float(np.sqrt(np.mean(err ** 2))) / rms
        report[key + "_raw"] = rel_err(gpu, ref)
        assert report[key + "_rms"] <= tol, (key, report)
        assert report[key + "_raw"] <= 8 * tol, (key, report)
        return
    raw = rel_err(gpu, ref)
    ex = rel_err_bf16(gpu, ref)
    report[key + "_raw"] = raw
    report[key] = ex
    report[key + "_floor"] = rounding_floor(ref)
    assert ex <= tol, (key, report)
    assert ex <= TIGHT[wdtype], (key, "beyond-rounding error above the tight bound", report)
    assert raw <= tol + report[key + "_floor"] * (1 + 1e-9), (key, report)
    if strict_raw is None:
        strict_raw = report[key + "_floor"] <= tol
    report[key + "_literal_asserted"] = bool(strict_raw)
    if strict_raw:
        assert raw <= tol, (key, "raw error above the literal bound", report)


def torch_bf16(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(device).contiguous()


def torch_bits(t) -> np.ndarray:
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


class _DeviceView:
    """A raw device pointer seen through __cuda_array_interface__."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def fetch(ptr: int, shape, dtype):
    """Copy a device buffer (raw pointer) to host numpy."""
    import torch
    dtype = np.dtype(dtype)
    code = {np.dtype(np.uint16): "<i2", np.dtype(np.int16): "<i2", np.dtype(np.float32): "<f4",
            np.dtype(np.int32): "<i4", np.dtype(np.uint8): "|u1"}[dtype]
    torch.cuda.synchronize()
    t = torch.as_tensor(_DeviceView(ptr, shape, code), device="cuda")
    return t.cpu().numpy().view(dtype).reshape(shape).copy()


def run_gpu_layer(layer, x_bits: np.ndarray, a_bits: np.ndarray, with_debug: bool = True) -> dict:
    """One kd_decode_layer call; returns output and intermediates as numpy."""
    import torch
    import moe_decode_layer_skinny_b200 as kd
    s = layer.spec
    M = x_bits.shape[0]
    hidden = torch_bf16(x_bits)
    attn = torch_bf16(a_bits)
    layer.decode(hidden, attn, M)
    torch.cuda.synchronize()
    layer.check()
    res = {"out": torch_bits(hidden)}
    nq = (s.q_heads + 2 * s.kv_heads) * s.head_dim
    res["qkv"] = fetch(layer.qkv_ptr(), (M, nq), np.uint16)
    if with_debug:
        res["h1"] = fetch(layer.debug_ptr(kd.T_H1F), (M, s.hidden), np.float32)
        res["logits"] = fetch(layer.debug_ptr(kd.T_LOGITS), (M, s.n_experts), np.float32)
        res["idx"] = fetch(layer.debug_ptr(kd.T_IDX), (M, s.top_k), np.int32)
        res["gates"] = fetch(layer.debug_ptr(kd.T_GATES), (M, s.top_k), np.float32)
        res["counts"] = fetch(layer.debug_ptr(kd.T_COUNTS), (s.n_experts,), np.int32)
        res["n_active"] = int(fetch(layer.debug_ptr(kd.T_NACTIVE), (1,), np.int32)[0])
    return res


def selection_check(gpu_idx: np.ndarray, ref_logits: np.ndarray, ref_idx: np.ndarray, k: int,
                    key_bias=None):
    """Tokens whose selections differ; each must be an excused near-tie (of
    the selection keys: the logits, plus key_bias for a selection-only bias)."""
    bad = []
    for t in range(gpu_idx.shape[0]):
        if set(gpu_idx[t].tolist()) == set(ref_idx[t].tolist()):
            continue
        keys = ref_logits[t] + (0 if key_bias is None else key_bias)
        srt = np.sort(keys)[::-1]
        gap = srt[k - 1] - srt[k] if len(srt) > k else np.inf
        assert gap < TIE_GAP, f"token {t}: selection {sorted(gpu_idx[t])} vs oracle " \
                              f"{sorted(ref_idx[t])}, gap {gap:.3g} not a near tie"
        bad.append(t)
    return bad


def compare_layer(dims, gpu: dict, x_bits, a_bits, *, wdtype=0, layer_id=0, seed=0, bias=None,
                  rows=None, check_qkv=True, strict_raw=None, bias_select_only=False,
                  routed_scale=1.0, tol_key=None) -> dict:
    """Compare one GPU layer call with the oracle (all rows, or the listed rows,
    each recomputed on its own -- rows are independent)."""
    x = bf16_to_f64(x_bits)
    a = bf16_to_f64(a_bits)
    rows = list(range(x.shape[0])) if rows is None else list(rows)
    var = dict(bias_select_only=bias_select_only, routed_scale=routed_scale)
    ref = oracle.layer(dims, x[rows], a[rows], wdtype=wdtype, layer_id=layer_id, seed=seed,
                       bias=bias, want_qkv=check_qkv, **var)
    g = {k: (v[rows] if isinstance(v, np.ndarray) and v.ndim >= 1 and k not in ("counts",) else v)
         for k, v in gpu.items()}
    report = {}
    if "idx" in g:
        excused = selection_check(g["idx"], ref["logits"], ref["idx"], dims.top_k,
                                  key_bias=bias if bias_select_only else None)
        report["excused"] = excused
        for t in excused:
            rf = oracle.layer(dims, x[rows][t:t + 1], a[rows][t:t + 1], wdtype=wdtype,
                              layer_id=layer_id, seed=seed, bias=bias,
                              forced_idx=g["idx"][t:t + 1], want_qkv=False, **var)
            ref["out"][t] = rf["out"][0]
            ref["gates"][t] = rf["gates"][0]
            ref["idx"][t] = rf["idx"][0]
        # gates by expert id
        for t in range(len(rows)):
            gm = dict(zip(g["idx"][t].tolist(), g["gates"][t].tolist()))
            for e, w in zip(ref["idx"][t].tolist(), ref["gates"][t].tolist()):
                assert abs(gm[e] - w) < 1e-4, (t, e, gm[e], w)
        report["h1"] = rel_err(g["h1"], ref["h1"])
        report["logits"] = rel_err(g["logits"], ref["logits"])
        assert report["h1"] < 1e-4, report
        assert report["logits"] < 1e-3, report
    tk = wdtype if tol_key is None else tol_key
    check_output(report, "out", bf16_to_f64(g["out"]), ref["out"], tk, strict_raw)
    if check_qkv:   # (the projections are the same for W8A8)
        check_output(report, "qkv", bf16_to_f64(g["qkv"]), ref["qkv"], wdtype, strict_raw)
    return report
