"""CUDA layer vs the CPU oracle, through the C ABI (libkd.so).

Covers the five workloads: the tiny layer at many token counts (bf16 and
FP8), the H=7168 layer at M=1 and at M=8 speculative-verify rows, the M=64
Zipf-biased layer on sampled rows plus whole-batch properties, and the
4-layer FP8 stack captured in a CUDA graph.
"""
import numpy as np
import pytest

import kdgen
import oracle
from kdgen import K2, TINY, WORKLOADS
from kdtest import (TOL, bf16_to_f64, compare_layer, fetch, rel_err_bf16, run_gpu_layer,
                    torch_bf16, torch_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kd(torch_cuda):
    import moe_decode_layer_skinny_b200 as kd
    kd.lib()
    return kd


def make_layer(kd, dims, wdtype=0, layer_id=0, bias=None, max_tokens=64, seed=0):
    spec = kd.LayerSpec.from_dims(dims, wdtype=wdtype, layer_id=layer_id, max_tokens=max_tokens,
                                  router_bias=bias)
    return kd.Layer(spec, seed=seed)


def inputs(dims, M, rho=0.0, seed=0, layer=0):
    x = kdgen.activations(seed, 0, kdgen.HIDDEN_IN, M, dims.hidden, rho)
    a = kdgen.activations(seed, layer, kdgen.ATTN_OUT, M, dims.attn, rho)
    return x, a


# ---------------------------------------------------------------- generator on device

@pytest.mark.parametrize("wdtype", [0, 1])
def test_device_weights_match_generator(kd, wdtype):
    d = TINY
    L = make_layer(kd, d, wdtype=wdtype)
    try:
        for kind, e, R, K in [(1, -1, d.nqkv, d.hidden), (2, -1, d.hidden, d.attn),
                              (3, -1, d.n_experts, d.hidden), (4, -1, d.inter, d.hidden),
                              (5, 3, d.inter, d.hidden), (6, 7, d.hidden, d.inter)]:
            slot = 0 if kind <= 3 or e < 0 else e + 1
            if wdtype == 0:
                ref = kdgen.weight_bf16(0, 0, kind, slot, R, K)
                assert np.array_equal(L.read_weight(kind, e, 0, R), ref)
            else:
                codes, scales = kdgen.weight_fp8(0, 0, kind, slot, R, K)
                c, s = L.read_weight(kind, e, 0, R)
                assert np.array_equal(c, codes)
                assert np.array_equal(s, scales)
    finally:
        L.close()


def test_device_weights_match_generator_k2_sampled(kd):
    L = make_layer(kd, K2, max_tokens=8)
    try:
        for kind, e, R, K, r0 in [(1, -1, K2.nqkv, K2.hidden, 10000), (2, -1, K2.hidden, K2.attn, 7000),
                                  (3, -1, K2.n_experts, K2.hidden, 250), (4, 255, K2.inter, K2.hidden, 2040),
                                  (5, 0, K2.inter, K2.hidden, 0), (6, 131, K2.hidden, K2.inter, 3000)]:
            slot = 0 if kind <= 3 or e < 0 else e + 1
            got = L.read_weight(kind, e, r0, 4)
            vals = kdgen.values(0, kdgen.uid(0, kind, slot), r0 * K, 4 * K, kdgen.W002)
            assert np.array_equal(got.reshape(-1), kdgen.to_bf16_bits(vals))
    finally:
        L.close()


# ---------------------------------------------------------------- tiny layer

@pytest.mark.parametrize("wdtype", [0, 1])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 13, 32, 64])
def test_tiny_layer_parity(kd, wdtype, M):
    d = TINY
    L = make_layer(kd, d, wdtype=wdtype)
    try:
        x, a = inputs(d, M, rho=0.5)
        g = run_gpu_layer(L, x, a)
        compare_layer(d, g, x, a, wdtype=wdtype)
        assert g["counts"].sum() == M * d.top_k
        assert g["n_active"] == int((g["counts"] > 0).sum())
    finally:
        L.close()


def test_tiny_variants(kd):
    # 512-wide QKV (2 kv heads), top-1, no shared expert, biased router
    from kdgen import Dims
    for d, bias in [(Dims(256, 4, 2, 64, 8, 2, 1, 128), None),
                    (Dims(256, 4, 1, 64, 8, 1, 0, 128), kdgen.zipf_bias(8, 1.1)),
                    (Dims(384, 2, 1, 128, 16, 4, 1, 256), kdgen.zipf_bias(16, 0.5))]:
        L = make_layer(kd, d, bias=bias)
        try:
            x, a = inputs(d, 7)
            g = run_gpu_layer(L, x, a)
            compare_layer(d, g, x, a, bias=None if bias is None else bias.astype(np.float64))
        finally:
            L.close()


def test_determinism_and_in_place(kd):
    import torch
    d = TINY
    L = make_layer(kd, d)
    try:
        x, a = inputs(d, 5)
        h1 = torch_bf16(x); h2 = torch_bf16(x); at = torch_bf16(a)
        L.decode(h1, at); L.decode(h2, at)
        torch.cuda.synchronize()
        assert torch.equal(h1, h2)
        assert not np.array_equal(torch_bits(h1), x)
        # only the first M rows are touched
        big = torch_bf16(np.concatenate([x, x]))
        L.decode(big, torch_bf16(np.concatenate([a, a])), 5)
        torch.cuda.synchronize()
        assert np.array_equal(torch_bits(big)[5:], x)
        assert torch.equal(big[:5], h1)
    finally:
        L.close()


def test_error_paths(kd):
    import torch
    d = TINY
    L = make_layer(kd, d, max_tokens=4)
    try:
        h = torch.zeros(8, d.hidden, dtype=torch.bfloat16, device="cuda")
        a = torch.zeros(8, d.attn, dtype=torch.bfloat16, device="cuda")
        for M in (0, 5, -1):
            with pytest.raises(kd.KdError) as ei:
                L.decode(h, a, M)
            assert ei.value.code == kd.KD_ERANGE
        assert kd.lib().kd_decode_layer(L.handle, None, a.data_ptr(), 1, None) == kd.KD_EINVAL
        L.decode(h, a, 4)
        L.check()
        # launches per call: CUDA-core path below 4 tokens, tensor-core path
        # (+ the combine launch) from 4; + the shared expert's gate/up
        assert L.launches(1) == 5 and L.launches(3) == 5
        assert L.launches(4) == 6
        with pytest.raises(kd.KdError) as ei:
            L.launches(5)
        assert ei.value.code == kd.KD_ERANGE
    finally:
        L.close()


# ---------------------------------------------------------------- H=7168 layers

@pytest.fixture(scope="module")
def k2_layer(kd):
    L = make_layer(kd, K2, max_tokens=64)
    yield L
    L.close()


def test_batch1_layer_parity(kd, k2_layer):
    w = WORKLOADS["batch1"]
    x, a = w.hidden_in(), w.attn_out()
    g = run_gpu_layer(k2_layer, x, a)
    r = compare_layer(K2, g, x, a)
    assert g["n_active"] == 8
    print("batch1", r)


def test_verify8_layer_parity(kd, k2_layer):
    w = WORKLOADS["verify8"]
    x, a = w.hidden_in(), w.attn_out()
    g = run_gpu_layer(k2_layer, x, a)
    r = compare_layer(K2, g, x, a)
    assert g["n_active"] < 8 * 8  # correlated rows share experts
    print("verify8", r, "active experts", g["n_active"])


@pytest.mark.parametrize("M", [2, 3, 16])
def test_k2_other_token_counts(kd, k2_layer, M):
    x, a = inputs(K2, M, seed=3)
    g = run_gpu_layer(k2_layer, x, a)
    compare_layer(K2, g, x, a, rows=[0, M - 1], check_qkv=True)


def test_batch64_zipf_parity_sampled(kd):
    w = WORKLOADS["batch64_zipf"]
    bias = w.bias()
    L = make_layer(kd, K2, bias=bias, max_tokens=64)
    try:
        x, a = w.hidden_in(), w.attn_out()
        g = run_gpu_layer(L, x, a)
        r = compare_layer(K2, g, x, a, bias=bias.astype(np.float64), rows=[0, 37, 63])
        # whole-batch properties
        M, k = 64, K2.top_k
        assert np.allclose(g["gates"].sum(1), 1.0, atol=1e-5)
        assert all(len(set(row)) == k for row in g["idx"].tolist())
        assert g["counts"].sum() == M * k
        # skewed load from the Zipf bias: the hottest experts are the low ids
        assert g["counts"].max() >= 4 * (M * k) / K2.n_experts
        assert g["counts"][:4].max() == g["counts"].max()
        # selected logits dominate the rest, per token
        for t in range(M):
            sel = g["logits"][t, g["idx"][t]]
            rest = np.delete(g["logits"][t], g["idx"][t])
            assert sel.min() >= rest.max()
        print("batch64_zipf", r, "active", g["n_active"], "max per expert", g["counts"].max())
    finally:
        L.close()


# ---------------------------------------------------------------- 4-layer FP8 stack

def test_stack4_fp8(kd):
    import torch
    w = WORKLOADS["stack4_fp8"]
    M, nl = w.M, w.n_layers
    layers = [make_layer(kd, K2, wdtype=1, layer_id=l, max_tokens=M) for l in range(nl)]
    try:
        x = w.hidden_in()
        attn = np.stack([w.attn_out(l) for l in range(nl)])
        # eager, layer by layer, keeping every intermediate
        hs = [x]
        h = torch_bf16(x)
        for l in range(nl):
            layers[l].decode(h, torch_bf16(attn[l]))
            torch.cuda.synchronize()
            layers[l].check()
            hs.append(torch_bits(h))
        # each layer against the oracle on sampled rows, given the GPU's input
        for l in range(nl):
            rows = [0, 17, 31] if l in (0, nl - 1) else [5]
            xl = bf16_to_f64(hs[l])[rows]
            al = bf16_to_f64(attn[l])[rows]
            ref = oracle.layer(K2, xl, al, wdtype=1, layer_id=l, want_qkv=False)
            err = rel_err_bf16(bf16_to_f64(hs[l + 1])[rows], ref["out"])
            assert err <= TOL[1], (l, err)
        # the graph-captured stack (with and without L2 prefetch) gives the
        # same bits as the eager sequence
        at = torch_bf16(attn.reshape(nl * M, -1))
        for pf in (True, False):
            st = kd.Stack(layers, M, prefetch=pf)
            hg = torch_bf16(x)
            st.run(hg, at)
            torch.cuda.synchronize()
            for L in layers:
                L.check()
            assert np.array_equal(torch_bits(hg), hs[-1])
            # replay with fresh input in the same buffers
            hg.copy_(torch_bf16(x))
            st.run(hg, at)
            torch.cuda.synchronize()
            assert np.array_equal(torch_bits(hg), hs[-1])
            st.close()
    finally:
        for L in layers:
            L.close()
