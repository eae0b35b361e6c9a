"""The full decode layer (RMSNorm, QKV with the KV-cache append, attention
over the FP8 e4m3 cache, o-proj + residual, RMSNorm, MoE) on the GPU through
kd_decode_layer_full, against the full-layer oracle.

Checks, per call: the e4m3 codes the GPU wrote for the new tokens equal the
oracle's, except where the oracle's value lies within 1e-4 (relative) of a
rounding midpoint (the GPU computes k in fp32, the oracle in fp64, and such
a value may round either way); every other cache entry is untouched.  The
rest is compared with the oracle run on the GPU's cache codes: the
attention output and h1 element by element, the router's selection exactly
(near ties excused as in the other parity tests), and the layer output and
qkv with the tolerances of the layer (1e-2 / 3e-2 of rms, bf16 weights /
FP8).  Token layouts: independent sequences at ragged positions, and one
sequence with consecutive positions (a speculative-verify step, causal).
"""
import numpy as np
import pytest

import kdgen
import oracle
from kdgen import K2, Dims
from kdtest import TIE_GAP, bf16_to_f64, check_output, fetch, rel_err, torch_bf16, torch_bits

pytestmark = pytest.mark.gpu

TINYF = Dims(hidden=256, q_heads=4, kv_heads=2, head_dim=64, n_experts=8, top_k=2, n_shared=1,
             inter=128)


@pytest.fixture(scope="module")
def kd(torch_cuda):
    import moe_decode_layer_skinny_b200 as kd
    kd.lib()
    return kd


def kv_scales(dims):
    # |k| ~ 0.02 sqrt(H) |u| with |u| ~ 1: the largest magnitudes near 448 codes
    sigma = 0.02 * np.sqrt(dims.hidden)
    return float(np.float32(4 * sigma / 448)), float(np.float32(4 * sigma / 448)), sigma


def make_full(kd, dims, n_seq, max_ctx, wdtype=0, max_tokens=8, layer_id=0, mma_min=0):
    ks, vs, _ = kv_scales(dims)
    spec = kd.LayerSpec.from_dims(dims, wdtype=wdtype, layer_id=layer_id, max_tokens=max_tokens,
                                  full_layer=1, kv_n_seq=n_seq, kv_max_ctx=max_ctx, k_scale=ks,
                                  v_scale=vs, mma_min_tokens=mma_min)
    return kd.Layer(spec, seed=0)


def cache_inputs(dims, n_seq, max_ctx, layer_id=0):
    ks, vs, sigma = kv_scales(dims)
    w = dims.kv_heads * dims.head_dim
    kc = kdgen.kv_cache(0, layer_id, kdgen.KCACHE, n_seq, max_ctx, w, sigma, ks)
    vc = kdgen.kv_cache(0, layer_id, kdgen.VCACHE, n_seq, max_ctx, w, sigma, vs)
    return kc, vc


def run_full(kd, layer, x_bits, kc0, vc0, seq, pos):
    import torch
    s = layer.spec
    M = x_bits.shape[0]
    hidden = torch_bf16(x_bits)
    kc = torch.from_numpy(kc0.copy()).cuda()
    vc = torch.from_numpy(vc0.copy()).cuda()
    st = torch.from_numpy(np.asarray(seq, np.int32)).cuda()
    pt = torch.from_numpy(np.asarray(pos, np.int32)).cuda()
    layer.decode_full(hidden, kc, vc, st, pt, M)
    torch.cuda.synchronize()
    layer.check()
    nq = (s.q_heads + 2 * s.kv_heads) * s.head_dim
    return {"out": torch_bits(hidden), "kc": kc.cpu().numpy(), "vc": vc.cpu().numpy(),
            "qkv": fetch(layer.qkv_ptr(), (M, nq), np.uint16),
            "attn": fetch(layer.debug_ptr(kd.T_ATTN), (M, s.q_heads * s.head_dim), np.float32),
            "h1": fetch(layer.debug_ptr(kd.T_RESID), (M, s.hidden), np.float32),
            "w": fetch(layer.debug_ptr(kd.T_H1F), (M, s.hidden), np.float32),
            "logits": fetch(layer.debug_ptr(kd.T_LOGITS), (M, s.n_experts), np.float32),
            "idx": fetch(layer.debug_ptr(kd.T_IDX), (M, s.top_k), np.int32),
            "gates": fetch(layer.debug_ptr(kd.T_GATES), (M, s.top_k), np.float32)}


def check_new_codes(gpu_c, ref_c, before, vals, seq, pos, width):
    """New positions: equal codes, or a near tie of the oracle's value;
    everything else untouched.  The GPU computes k and v in fp32 from bf16
    hi + lo activations (~16 significant bits), so its value of an element
    is off by up to ~1e-5 of the row's rms; a code may differ where the
    oracle's value lies within 1e-4 x rms(row) of a rounding midpoint."""
    mask = np.zeros(gpu_c.shape[:2], bool)
    mask[np.asarray(seq), np.asarray(pos)] = True
    assert np.array_equal(gpu_c[~mask], before[~mask])
    dec = np.vectorize(oracle.e4m3_value)
    n_tie = 0
    for t, (s, p) in enumerate(zip(seq, pos)):
        g, r = gpu_c[s, p], ref_c[s, p]
        bad = np.nonzero(g != r)[0]
        scale = float(np.sqrt(np.mean(vals[t] ** 2)))
        for i in bad:
            v = vals[t][i]
            a, b = dec(g[i]), dec(r[i])
            mid = (a + b) / 2
            assert abs(v - mid) <= 1e-4 * scale, (t, i, v, a, b, scale)
            n_tie += 1
    return n_tie


def compare_full(dims, g, x_bits, kc0, vc0, seq, pos, wdtype):
    ks, vs, _ = kv_scales(dims)
    x = bf16_to_f64(x_bits)
    M = x.shape[0]
    own = oracle.layer_full(dims, x, kc0, vc0, ks, vs, seq, pos, wdtype=wdtype)
    qw, kw = dims.q_heads * dims.head_dim, dims.kv_heads * dims.head_dim
    kvals = own["qkv"][:, qw:qw + kw] / ks
    vvals = own["qkv"][:, qw + kw:] / vs
    report = {"kv_ties": check_new_codes(g["kc"], own["kc"], kc0, kvals, seq, pos, kw) +
              check_new_codes(g["vc"], own["vc"], vc0, vvals, seq, pos, kw)}
    ref = oracle.layer_full(dims, x, g["kc"], g["vc"], ks, vs, seq, pos, wdtype=wdtype,
                            keep_new_kv=True)
    # intermediate fp32 tensors: q, k, v come from bf16 hi + lo activations
    # (~2^-16 relative) with fp32 accumulation; scores of magnitude ~10 carry
    # that error into the softmax weights, ~1e-4 of the attention output
    report["attn"] = rel_err(g["attn"], ref["attn"])
    report["h1"] = rel_err(g["h1"], ref["h1"])
    report["w"] = rel_err(g["w"], ref["v"])
    assert report["attn"] < 1e-3, report
    assert report["h1"] < 1e-3, report
    assert report["w"] < 1e-3, report
    # selection: exact unless a near tie, then that row under the GPU's selection
    for t in range(M):
        if set(g["idx"][t].tolist()) == set(ref["idx"][t].tolist()):
            continue
        srt = np.sort(ref["logits"][t])[::-1]
        assert srt[dims.top_k - 1] - srt[dims.top_k] < TIE_GAP, (t, g["idx"][t], ref["idx"][t])
        rf = oracle.layer_full(dims, x, g["kc"], g["vc"], ks, vs, seq, pos, wdtype=wdtype,
                               keep_new_kv=True, forced_idx=g["idx"])
        ref["out"][t], ref["gates"][t], ref["idx"][t] = rf["out"][t], rf["gates"][t], rf["idx"][t]
    for t in range(M):
        gm = dict(zip(g["idx"][t].tolist(), g["gates"][t].tolist()))
        for e, wv in zip(ref["idx"][t].tolist(), ref["gates"][t].tolist()):
            assert abs(gm[e] - wv) < 1e-4, (t, e, gm[e], wv)
    check_output(report, "out", bf16_to_f64(g["out"]), ref["out"], wdtype)
    check_output(report, "qkv", bf16_to_f64(g["qkv"]), ref["qkv"], wdtype)
    return report


LAYOUTS = {
    # token -> (sequence, position): ragged independent sequences, and one
    # sequence at consecutive positions (verify step)
    "ragged": lambda M, n_seq, ctx: ([t % n_seq for t in range(M)],
                                     [(37 * t + 11) % ctx for t in range(M)]),
    "verify": lambda M, n_seq, ctx: ([n_seq - 1] * M, [ctx - M + t for t in range(M)]),
}


@pytest.mark.parametrize("wdtype", [0, 1])
@pytest.mark.parametrize("M", [1, 3, 5, 8])
@pytest.mark.parametrize("layout", ["ragged", "verify"])
def test_full_tiny(kd, wdtype, M, layout):
    """Tiny dims (2 kv heads of 2 query heads, head_dim 64), a 300-position
    cache (ten attention chunks), both engines (the CUDA-core kernels for
    M = 1 and 3, the tensor cores for 5 and 8)."""
    n_seq, ctx = 3, 300
    L = make_full(kd, TINYF, n_seq, ctx, wdtype=wdtype, mma_min=4)
    try:
        x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, TINYF.hidden, 0.3)
        kc0, vc0 = cache_inputs(TINYF, n_seq, ctx)
        seq, pos = LAYOUTS[layout](M, n_seq, ctx)
        g = run_full(kd, L, x, kc0, vc0, seq, pos)
        r = compare_full(TINYF, g, x, kc0, vc0, seq, pos, wdtype)
        print(layout, M, wdtype, r)
    finally:
        L.close()


@pytest.mark.parametrize("M,layout", [(1, "ragged"), (8, "verify"), (5, "ragged")])
def test_full_k2(kd, M, layout):
    """H=7168 layer with 64 query heads over 8 kv heads (head_dim 128), a
    2048-position cache; all rows against the oracle."""
    n_seq, ctx = 4, 2048
    L = make_full(kd, K2, n_seq, ctx, max_tokens=8)
    try:
        x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, K2.hidden, 0.9 if layout == "verify" else 0)
        kc0, vc0 = cache_inputs(K2, n_seq, ctx)
        seq, pos = LAYOUTS[layout](M, n_seq, ctx)
        g = run_full(kd, L, x, kc0, vc0, seq, pos)
        r = compare_full(K2, g, x, kc0, vc0, seq, pos, 0)
        print("k2", layout, M, r)
    finally:
        L.close()


def test_full_bad_position_is_reported(kd):
    """An out-of-range position: the token's attention is zero, nothing is
    written out of bounds, kd_layer_check reports KD_EDEVICE, and the next
    call is correct."""
    import torch
    n_seq, ctx = 2, 64
    L = make_full(kd, TINYF, n_seq, ctx)
    try:
        x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, 2, TINYF.hidden, 0.0)
        kc0, vc0 = cache_inputs(TINYF, n_seq, ctx)
        hidden = torch_bf16(x)
        kc = torch.from_numpy(kc0.copy()).cuda()
        vc = torch.from_numpy(vc0.copy()).cuda()
        seq = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
        pos = torch.tensor([5, ctx], dtype=torch.int32, device="cuda")   # token 1 out of range
        L.decode_full(hidden, kc, vc, seq, pos, 2)
        torch.cuda.synchronize()
        with pytest.raises(kd.KdError) as ei:
            L.check()
        assert ei.value.code == kd.KD_EDEVICE
        attn = fetch(L.debug_ptr(kd.T_ATTN), (2, TINYF.attn), np.float32)
        assert np.all(attn[1] == 0)
        assert np.array_equal(kc.cpu().numpy()[1], kc0[1])
        L.check()   # cleared
        g = run_full(kd, L, x, kc0, vc0, [0, 1], [5, 9])
        compare_full(TINYF, g, x, kc0, vc0, [0, 1], [5, 9], 0)
    finally:
        L.close()


def test_full_layer_entry_point_errors(kd):
    import torch
    L = kd.Layer(kd.LayerSpec.from_dims(TINYF, max_tokens=4), seed=0)   # not a full layer
    try:
        h = torch.zeros(4, TINYF.hidden, dtype=torch.bfloat16, device="cuda")
        c = torch.zeros(1, 8, TINYF.kv_heads * TINYF.head_dim, dtype=torch.uint8, device="cuda")
        i = torch.zeros(4, dtype=torch.int32, device="cuda")
        with pytest.raises(kd.KdError) as ei:
            L.decode_full(h, c, c, i, i, 1)
        assert ei.value.code == kd.KD_EINVAL
    finally:
        L.close()
    L = make_full(kd, TINYF, 1, 8, max_tokens=4)
    try:
        with pytest.raises(kd.KdError) as ei:
            L.decode_full(h, c, c, i, i, 5)
        assert ei.value.code == kd.KD_ERANGE
        assert L.launches(1) == 10 and L.launches(3) == 10
    finally:
        L.close()


def test_create_allocation_failure_releases_everything(kd):
    """Failure detection on the host: the n-th device allocation of
    kd_layer_create fails (test hook); the call returns KD_ENOMEM and the
    device's free memory is what it was (nothing leaked)."""
    import os
    import torch
    dims = Dims(hidden=1024, q_heads=8, kv_heads=2, head_dim=128, n_experts=16, top_k=4,
                n_shared=1, inter=512)
    spec = kd.LayerSpec.from_dims(dims, max_tokens=8, full_layer=1, kv_n_seq=2, kv_max_ctx=256,
                                  k_scale=0.01, v_scale=0.01)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    try:
        for n in (1, 3, 8, 20, 45):
            os.environ["KD_TEST_FAIL_ALLOC_AT"] = str(n)
            with pytest.raises(kd.KdError) as ei:
                kd.Layer(spec, seed=0)
            assert ei.value.code == kd.KD_ENOMEM
            assert "injected" in str(ei.value)
            torch.cuda.synchronize()
            assert abs(torch.cuda.mem_get_info()[0] - free0) < (1 << 20), n
    finally:
        os.environ.pop("KD_TEST_FAIL_ALLOC_AT", None)
    L = kd.Layer(spec, seed=0)   # and without the hook it is created
    L.close()
