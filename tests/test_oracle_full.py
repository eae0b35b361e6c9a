"""Pins of the full-layer oracle (RMSNorm, attention over an FP8 e4m3 KV
cache, pre-norm residual layer) against library routines and closed forms:
torch's float8_e4m3fn conversion, torch's RMSNorm, torch's scaled
dot-product attention, and cases whose answer is known without computing
the layer (a one-position context returns its value row, equal keys average
the values, zero projections return the input).

The attention half of the decode step is the part the write-ups describe as
attention with an FP8 KV cache (bigchange.ai "where the time went") fed by
the attention input projections (wireai.ir "4 key changes", item 1).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import kdgen
import oracle
from kdgen import Dims

TINYF = Dims(hidden=256, q_heads=4, kv_heads=2, head_dim=64, n_experts=8, top_k=2, n_shared=1,
             inter=128)


def e4m3_codes(v: np.ndarray) -> np.ndarray:
    """The oracle's encoder on each element (itself pinned against torch's
    float8_e4m3fn conversion below)."""
    v = np.asarray(v, np.float64)
    return np.array([oracle.e4m3_code(float(a)) for a in v.ravel()], np.uint8).reshape(v.shape)


def dec_torch(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


# ------------------------------------------------------------------ e4m3 encoder

def test_e4m3_encoder_matches_torch():
    # on fp32-exact inputs (torch converts float64 through float32, which
    # rounds twice; the oracle rounds the exact value once): every
    # representable value, the midpoints between neighbours (ties to even),
    # the fp32 neighbours of each midpoint, and random values of all scales
    rng = np.random.default_rng(1)
    reps = np.unique(np.abs(dec_torch(np.arange(256))[~np.isnan(dec_torch(np.arange(256)))]))
    mids = ((reps[1:] + reps[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([reps.astype(np.float32), mids, np.nextafter(mids, np.float32(np.inf)),
                           np.nextafter(mids, np.float32(0)),
                           (np.exp(rng.uniform(-14, 6, 20000)) * rng.choice([-1, 1], 20000))
                           .astype(np.float32)])
    vals = np.concatenate([vals, -vals])
    ours = np.array([oracle.e4m3_code(float(v)) for v in vals], np.uint8)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    # a value above a midpoint by less than fp32 can hold rounds up
    assert oracle.e4m3_code(1.0625 * (1 + 1e-12)) == 0x39 and oracle.e4m3_code(1.0625) == 0x38


def test_e4m3_encoder_saturates():
    for v in (448.0, 448.5, 470.0, 1e6):
        assert oracle.e4m3_code(v) == 0x7E and oracle.e4m3_code(-v) == 0xFE


# ------------------------------------------------------------------ RMSNorm

def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 384)) * np.array([1e-3, 1, 7, 100, 1e4])[:, None]
    g = 1 + 0.02 * rng.standard_normal(384)
    ref = F.rms_norm(torch.from_numpy(x), (384,), torch.from_numpy(g), eps=1e-6).numpy()
    assert np.allclose(oracle.rmsnorm(x, g, 1e-6), ref, rtol=1e-13, atol=0)


def test_rmsnorm_closed_forms():
    g = np.linspace(0.5, 1.5, 64)
    # a constant row c: every element becomes sign(c) * g * |c| / sqrt(c^2 + eps)
    for c in (3.0, -0.25):
        y = oracle.rmsnorm(np.full((1, 64), c), g, 1e-6)[0]
        assert np.allclose(y, np.sign(c) * g * abs(c) / math.sqrt(c * c + 1e-6), rtol=1e-15)
    # scale invariance (eps = 0)
    x = np.random.default_rng(3).standard_normal((1, 64))
    assert np.allclose(oracle.rmsnorm(17 * x, g, 0.0), oracle.rmsnorm(x, g, 0.0), rtol=1e-14)


# ------------------------------------------------------------------ attention

def _cache(rng, n_seq, ctx, width):
    return (rng.integers(0, 256, (n_seq, ctx, width)).astype(np.uint8) & 0xF7 | 0x30).astype(np.uint8)


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(4)
    hq, hkv, hd, n_seq, ctx = 8, 2, 32, 3, 40
    kc = _cache(rng, n_seq, ctx, hkv * hd)
    vc = _cache(rng, n_seq, ctx, hkv * hd)
    seq = np.array([2, 0, 1, 2, 0])
    pos = np.array([39, 0, 17, 5, 26])
    q = rng.standard_normal((5, hq * hd))
    ks, vs = 0.05, 0.2
    ours = oracle.attention(q, kc, vc, ks, vs, hq, hkv, hd, seq, pos)
    K = dec_torch(kc) * ks
    V = dec_torch(vc) * vs
    for t in range(5):
        L = pos[t] + 1
        qt = torch.from_numpy(q[t].reshape(1, hq, 1, hd))
        kt = torch.from_numpy(K[seq[t], :L].reshape(L, hkv, hd)).permute(1, 0, 2)
        vt = torch.from_numpy(V[seq[t], :L].reshape(L, hkv, hd)).permute(1, 0, 2)
        kt = kt.repeat_interleave(hq // hkv, 0)[None]
        vt = vt.repeat_interleave(hq // hkv, 0)[None]
        ref = F.scaled_dot_product_attention(qt, kt, vt).reshape(hq * hd).numpy()
        assert np.allclose(ours[t], ref, rtol=1e-12, atol=1e-14), t


def test_attention_closed_forms():
    rng = np.random.default_rng(5)
    hq, hkv, hd = 4, 1, 16
    kc = _cache(rng, 1, 9, hd)
    vc = _cache(rng, 1, 9, hd)
    q = rng.standard_normal((2, hq * hd))
    # one position: every head returns that position's value row
    o = oracle.attention(q, kc, vc, 0.1, 0.3, hq, hkv, hd, [0, 0], [0, 0])
    for h in range(hq):
        assert np.array_equal(o[0, h * hd:(h + 1) * hd], dec_torch(vc[0, 0]) * 0.3)
    # all keys equal: uniform weights, the mean of the value rows
    kc2 = np.repeat(kc[:, :1], 9, axis=1)
    o = oracle.attention(q[:1], kc2, vc, 0.1, 0.3, hq, hkv, hd, [0], [8])
    assert np.allclose(o[0, :hd], (dec_torch(vc[0]) * 0.3).mean(0), rtol=1e-13)


def test_attention_head_groups():
    # q head h reads kv head h // (hq / hkv): swapping the two kv heads'
    # caches swaps the two halves of the output
    rng = np.random.default_rng(6)
    hq, hkv, hd = 4, 2, 8
    kc = _cache(rng, 1, 5, hkv * hd)
    vc = _cache(rng, 1, 5, hkv * hd)
    q = rng.standard_normal((1, hq * hd))
    o = oracle.attention(q, kc, vc, 0.1, 0.1, hq, hkv, hd, [0], [4])
    sw = lambda c: np.concatenate([c[..., hd:], c[..., :hd]], -1)
    qs = np.concatenate([q[:, 2 * hd:], q[:, :2 * hd]], 1)
    o2 = oracle.attention(qs, sw(kc), sw(vc), 0.1, 0.1, hq, hkv, hd, [0], [4])
    assert np.allclose(np.concatenate([o2[:, 2 * hd:], o2[:, :2 * hd]], 1), o, rtol=1e-14)


# ------------------------------------------------------------------ full layer

def _full_inputs(dims, M, n_seq, ctx, seed=0, k_scale=0.01, v_scale=0.01):
    x = kdgen.bf16_bits_to_f32(kdgen.activations(seed, 0, kdgen.HIDDEN_IN, M, dims.hidden, 0.0))
    w = dims.kv_heads * dims.head_dim
    kc = kdgen.kv_cache(seed, 0, kdgen.KCACHE, n_seq, ctx, w, 1.0, k_scale)
    vc = kdgen.kv_cache(seed, 0, kdgen.VCACHE, n_seq, ctx, w, 1.0, v_scale)
    return x.astype(np.float64), kc, vc


def _gen_weights(dims):
    from test_oracle_pins import explicit_weights
    w = explicit_weights(dims)
    w["g1"] = kdgen.bf16_bits_to_f32(kdgen.norm_bf16(0, 0, kdgen.NORM1, dims.hidden)).astype(np.float64)
    w["g2"] = kdgen.bf16_bits_to_f32(kdgen.norm_bf16(0, 0, kdgen.NORM2, dims.hidden)).astype(np.float64)
    return w


def test_full_layer_against_torch_composition():
    """The full layer recomposed from library routines (torch matmuls,
    RMSNorm, float8 conversion, SDPA, top-k) on the tiny dims."""
    d = TINYF
    M, n_seq, ctx = 3, 2, 12
    x, kc, vc = _full_inputs(d, M, n_seq, ctx)
    seq, pos = np.array([1, 0, 1]), np.array([7, 11, 8])
    ks, vs = 0.01, 0.01
    r = oracle.layer_full(d, x, kc, vc, ks, vs, seq, pos)
    W = {k: torch.from_numpy(v) for k, v in _gen_weights(d).items()}
    X = torch.from_numpy(x)
    u = F.rms_norm(X, (d.hidden,), W["g1"], eps=1e-6)
    qkv = u @ W["wqkv"].T
    hq, hkv, hd = d.q_heads, d.kv_heads, d.head_dim
    q, k, v = qkv[:, :hq * hd], qkv[:, hq * hd:(hq + hkv) * hd], qkv[:, (hq + hkv) * hd:]
    kc2, vc2 = kc.copy(), vc.copy()
    for t in range(M):
        kc2[seq[t], pos[t]] = e4m3_codes((k[t] / ks).numpy())
        vc2[seq[t], pos[t]] = e4m3_codes((v[t] / vs).numpy())
    assert np.array_equal(r["kc"], kc2) and np.array_equal(r["vc"], vc2)
    K = torch.from_numpy(dec_torch(kc2) * ks)
    V = torch.from_numpy(dec_torch(vc2) * vs)
    a = torch.zeros(M, hq * hd, dtype=torch.float64)
    for t in range(M):
        L = pos[t] + 1
        kt = K[seq[t], :L].reshape(L, hkv, hd).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)
        vt = V[seq[t], :L].reshape(L, hkv, hd).permute(1, 0, 2).repeat_interleave(hq // hkv, 0)
        a[t] = F.scaled_dot_product_attention(q[t].reshape(hq, 1, hd)[None], kt[None],
                                              vt[None]).reshape(-1)
    h1 = X + a @ W["wo"].T
    vv = F.rms_norm(h1, (d.hidden,), W["g2"], eps=1e-6)
    lg = vv @ W["wr"].T
    gv, gi = torch.topk(lg, d.top_k, dim=1)
    gates = torch.softmax(gv, dim=1)

    def swiglu(e, z):  # e = 0: shared, 1 + routed id
        return (F.silu(z @ W["wg"][e].T) * (z @ W["wu"][e].T)) @ W["wd"][e].T

    out = h1 + swiglu(0, vv)
    for t in range(M):
        for j in range(d.top_k):
            out[t] += gates[t, j] * swiglu(1 + int(gi[t, j]), vv[t:t + 1])[0]
    assert np.allclose(r["attn"], a.numpy(), rtol=1e-11, atol=1e-13)
    assert np.allclose(r["h1"], h1.numpy(), rtol=1e-11, atol=1e-12)
    assert np.array_equal(r["idx"], gi.numpy())
    assert np.allclose(r["out"], out.numpy(), rtol=1e-10, atol=1e-11)


def test_full_layer_closed_form_zero_projections():
    """Wo = 0 and every down projection 0: the output is the input."""
    d = TINYF
    x, kc, vc = _full_inputs(d, 2, 1, 6)
    w = _gen_weights(d)
    w["wo"] = np.zeros_like(w["wo"])
    w["wd"] = np.zeros_like(w["wd"])
    r = oracle.layer_full(d, x, kc, vc, 0.01, 0.01, [0, 0], [4, 5], weights=w)
    assert np.array_equal(r["out"], x)


def test_full_layer_verify_step_is_causal():
    """Tokens of one sequence at consecutive positions: the first token's
    result does not depend on the later ones (they are written after it in
    position), and each later token sees the earlier tokens' keys."""
    d = TINYF
    x, kc, vc = _full_inputs(d, 4, 1, 10)
    full = oracle.layer_full(d, x, kc, vc, 0.01, 0.01, [0] * 4, [5, 6, 7, 8])
    first = oracle.layer_full(d, x[:1], kc, vc, 0.01, 0.01, [0], [5])
    assert np.array_equal(full["out"][0], first["out"][0])
    assert np.array_equal(full["kc"][0, 5], first["kc"][0, 5])
    # the last token with the first three written in a previous call
    pre = oracle.layer_full(d, x[:3], kc, vc, 0.01, 0.01, [0] * 3, [5, 6, 7])
    last = oracle.layer_full(d, x[3:], pre["kc"], pre["vc"], 0.01, 0.01, [0], [8])
    assert np.allclose(full["out"][3], last["out"][0], rtol=1e-14, atol=1e-15)


def test_full_layer_keep_new_kv():
    d = TINYF
    x, kc, vc = _full_inputs(d, 2, 2, 6)
    r = oracle.layer_full(d, x, kc, vc, 0.01, 0.01, [0, 1], [3, 5])
    r2 = oracle.layer_full(d, x, r["kc"], r["vc"], 0.01, 0.01, [0, 1], [3, 5], keep_new_kv=True)
    assert np.array_equal(r["out"], r2["out"])
