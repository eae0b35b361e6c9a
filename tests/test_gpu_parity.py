"""CUDA layer vs the CPU oracle, through the C ABI (libkd.so).

Covers the five workloads, every row of every output compared element by
element with the oracle: the tiny layer at many token counts (bf16 and FP8),
the H=7168 layer at M=1, at the speculative-verify shapes M=4..8 (3-7 draft
tokens + 1) and at M=2, 3, 16, the M=64 Zipf-biased layer, and the 4-layer
FP8 stack (each layer against the oracle given the GPU's input to it, then
the CUDA-graph replay against the eager chain); plus exact router ties
through the allocation-free router entry point.

Oracle wall times (fp64, all host threads; 8 cores of a 2.7 GHz Xeon): the
M=1 layer ~0.3 s, M=4..16 ~0.5-1.5 s each, the M=64 Zipf layer ~11 s, one
FP8 layer of the stack ~50 s (FP8 weights are generated twice per 128x128
block: once for the block's amax, once to quantise).
"""
import numpy as np
import pytest

import kdgen
import oracle
from kdgen import K2, TINY, WORKLOADS
from kdtest import (TOL, bf16_to_f64, compare_layer, fetch, rel_err_bf16, run_gpu_layer,
                    selection_check, torch_bf16, torch_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kd(torch_cuda):
    import moe_decode_layer_skinny_b200 as kd
    kd.lib()
    return kd


# engines: "tensor" = the default (tcgen05 kernels for every M), "cores" =
# the CUDA-core streaming kernels (mma_min_tokens beyond any M)
ENGINE_MMA_MIN = {"tensor": 0, "cores": 1000}


def make_layer(kd, dims, wdtype=0, layer_id=0, bias=None, max_tokens=64, seed=0, engine="tensor"):
    spec = kd.LayerSpec.from_dims(dims, wdtype=wdtype, layer_id=layer_id, max_tokens=max_tokens,
                                  router_bias=bias, mma_min_tokens=ENGINE_MMA_MIN[engine])
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
@pytest.mark.parametrize("M,engine", [(1, "tensor"), (2, "tensor"), (3, "tensor"), (5, "tensor"),
                                      (8, "tensor"), (13, "tensor"), (32, "tensor"), (64, "tensor"),
                                      (1, "cores"), (2, "cores"), (3, "cores"), (5, "cores")])
def test_tiny_layer_parity(kd, wdtype, M, engine):
    d = TINY
    L = make_layer(kd, d, wdtype=wdtype, engine=engine)
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


@pytest.mark.parametrize("wdtype", [0, 1])
@pytest.mark.parametrize("M,engine", [(3, "cores"), (8, "tensor"), (2, "tensor")])
def test_gating_variants(kd, wdtype, M, engine):
    """Selection-only router bias (the gates from the unbiased logits) and a
    routed scaling factor, on both engines."""
    d = TINY
    bias = kdgen.zipf_bias(d.n_experts, 1.1)
    for sel, rs in [(1, 1.0), (0, 2.5), (1, 0.75)]:
        spec = kd.LayerSpec.from_dims(d, wdtype=wdtype, max_tokens=8, router_bias=bias,
                                      bias_select_only=sel, routed_scale=rs,
                                      mma_min_tokens=ENGINE_MMA_MIN[engine])
        L = kd.Layer(spec, seed=0)
        try:
            x, a = inputs(d, M, rho=0.3)
            g = run_gpu_layer(L, x, a)
            compare_layer(d, g, x, a, wdtype=wdtype, bias=bias.astype(np.float64),
                          bias_select_only=bool(sel), routed_scale=rs)
        finally:
            L.close()


@pytest.mark.parametrize("E,k,M,sel", [(384, 8, 8, 1), (384, 8, 40, 0), (640, 16, 5, 1),
                                        (1024, 16, 64, 0)])
def test_wide_router_layers(kd, E, k, M, sel):
    """More experts than 256 (a lane of the selection holds 16 or 32 logits),
    top-16, up to 64 tokens: the layer against the oracle, on the CUDA-core
    router (M <= 8) and the tensor-core router, with a selection-only or a
    logit bias.  Every row; the oracle takes 0.02-0.11 s per case."""
    from kdgen import Dims
    d = Dims(hidden=256, q_heads=2, kv_heads=1, head_dim=128, n_experts=E, top_k=k, n_shared=1,
             inter=128)
    bias = kdgen.zipf_bias(E, 0.3)
    spec = kd.LayerSpec.from_dims(d, max_tokens=64, router_bias=bias, bias_select_only=sel)
    L = kd.Layer(spec, seed=3)
    try:
        x, a = inputs(d, M, rho=0.2, seed=5)
        g = run_gpu_layer(L, x, a)
        compare_layer(d, g, x, a, seed=3, bias=bias.astype(np.float64), bias_select_only=bool(sel))
    finally:
        L.close()


@pytest.mark.parametrize("dims,M,rows", [(TINY, 8, None), (K2, 32, [0, 7, 19, 31])])
def test_w8a8_experts(kd, dims, M, rows):
    """FP8 expert weights with one e4m3 term per activation (W8A8) on the
    tensor cores: the output's rms error within one e4m3 rounding (2^-4) of
    its rms; the same selection; the projections as with two terms."""
    spec = kd.LayerSpec.from_dims(dims, wdtype=1, max_tokens=M, fp8_act_terms=1)
    L = kd.Layer(spec, seed=0)
    try:
        x, a = inputs(dims, M, rho=0.3)
        g = run_gpu_layer(L, x, a)
        r = compare_layer(dims, g, x, a, wdtype=1, rows=rows, tol_key=2)
        print("w8a8", dims.hidden, M, r)
    finally:
        L.close()
    with pytest.raises(kd.KdError) as e:
        kd.Layer(kd.LayerSpec.from_dims(TINY, wdtype=1, max_tokens=4, fp8_act_terms=3))
    assert e.value.code == kd.KD_EINVAL


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
        # launches per call: projections, router, gate/up, down, combine, +
        # the shared expert's gate/up, on either path
        assert L.launches(1) == 6 and L.launches(2) == 6
        assert L.launches(3) == 6 and L.launches(4) == 6
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
    r = compare_layer(K2, g, x, a, strict_raw=True)   # floor 0.0099 at this input
    assert g["n_active"] == 8
    print("batch1", r)


def test_k2_cuda_core_engine(kd):
    """The CUDA-core streaming kernels (mma_min_tokens beyond any M) on the
    H=7168 layer: batch 1, and two tokens; every row against the oracle."""
    L = make_layer(kd, K2, max_tokens=2, engine="cores")
    try:
        w = WORKLOADS["batch1"]
        x, a = w.hidden_in(), w.attn_out()
        g = run_gpu_layer(L, x, a)
        r = compare_layer(K2, g, x, a, strict_raw=True)   # floor 0.0099 at this input
        assert g["n_active"] == 8
        print("batch1 cores", r)
        x, a = inputs(K2, 2, seed=3)
        g = run_gpu_layer(L, x, a)
        print("M=2 cores", compare_layer(K2, g, x, a))
    finally:
        L.close()


def test_verify8_layer_parity(kd, k2_layer):
    w = WORKLOADS["verify8"]
    x, a = w.hidden_in(), w.attn_out()
    g = run_gpu_layer(k2_layer, x, a)
    r = compare_layer(K2, g, x, a)
    assert g["n_active"] < 8 * 8  # correlated rows share experts
    print("verify8", r, "active experts", g["n_active"])


@pytest.mark.parametrize("M", [2, 3, 4, 5, 6, 7, 16])
def test_k2_other_token_counts(kd, k2_layer, M):
    """All rows at M = 2, 3, 4..7 (speculative verify with 3..6 draft tokens
    + 1, correlated rows) and 16."""
    x, a = inputs(K2, M, seed=3, rho=0.9 if 4 <= M <= 7 else 0.0)
    g = run_gpu_layer(k2_layer, x, a)
    r = compare_layer(K2, g, x, a, check_qkv=True)
    assert g["counts"].sum() == M * K2.top_k
    print(f"M={M}", r)


def test_batch64_zipf_parity(kd):
    """All 64 rows against the oracle (~11 s of oracle time), plus whole-batch
    properties of the routing."""
    w = WORKLOADS["batch64_zipf"]
    bias = w.bias()
    L = make_layer(kd, K2, bias=bias, max_tokens=64)
    try:
        x, a = w.hidden_in(), w.attn_out()
        g = run_gpu_layer(L, x, a)
        r = compare_layer(K2, g, x, a, bias=bias.astype(np.float64))
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
    """Every row of every layer (out and qkv) against the oracle given the
    GPU's own input to that layer (~50 s of oracle time per layer), then the
    CUDA-graph stack, with and without L2 prefetch, against the eager chain."""
    import torch
    w = WORKLOADS["stack4_fp8"]
    M, nl = w.M, w.n_layers
    layers = [make_layer(kd, K2, wdtype=1, layer_id=l, max_tokens=M) for l in range(nl)]
    try:
        x = w.hidden_in()
        attn = np.stack([w.attn_out(l) for l in range(nl)])
        # eager, layer by layer, keeping every layer's input and output
        hs = [x]
        for l in range(nl):
            g = run_gpu_layer(layers[l], hs[l], attn[l])
            r = compare_layer(K2, g, hs[l], attn[l], wdtype=1, layer_id=l, check_qkv=True)
            print(f"stack layer {l}", r)
            hs.append(g["out"])
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


# ---------------------------------------------------------------- exact router ties

def tie_case(rng, H=256, E=16, k=4, M=5):
    """Router rows and fp32 h1 rows whose logits contain exact ties: rows
    2 and 13 are the same (the two largest logits), rows 6 and 11 are the
    same and rank k-1 / k (the selection boundary), rows 1 and 9 are the same
    lower down.  The other rows are scaled copies of one direction plus
    noise, so the order is the same for every token."""
    v = rng.standard_normal(H).astype(np.float32)
    alpha = np.linspace(-1.0, 1.0, E).astype(np.float32)
    alpha[[2, 13]] = 3.0
    alpha[3] = 2.5
    alpha[[6, 11]] = 2.0
    alpha[[1, 9]] = -0.5
    W = 0.01 * (alpha[:, None] * v[None, :] + 0.01 * rng.standard_normal((E, H)).astype(np.float32))
    Wb = kdgen.to_bf16_bits(W)
    Wb[13] = Wb[2]
    Wb[11] = Wb[6]
    Wb[9] = Wb[1]
    h1 = (v[None, :] + 0.3 * rng.standard_normal((M, H))).astype(np.float32)
    return Wb, h1


def oracle_router(Wb, h1, k, bias=None):
    """The oracle's top-k and gates for router weights Wb (bf16 bits) and h1:
    the layer with Wo = 0 (so h1 = x), zero experts and zero QKV."""
    from kdgen import Dims
    E, H = Wb.shape
    M = h1.shape[0]
    d = Dims(hidden=H, q_heads=1, kv_heads=0, head_dim=128, n_experts=E, top_k=k, n_shared=0,
             inter=128)
    weights = {"wqkv": np.zeros((d.nqkv, H)), "wo": np.zeros((H, d.attn)),
               "wr": bf16_to_f64(Wb), "wg": np.zeros((E, 128, H)), "wu": np.zeros((E, 128, H)),
               "wd": np.zeros((E, H, 128))}
    return d, oracle.layer(d, h1.astype(np.float64), np.zeros((M, d.attn)), weights=weights,
                           bias=bias)


def test_router_exact_ties_against_oracle(kd):
    """Exact ties go to the lower expert id, on the GPU as in the oracle."""
    import torch
    rng = np.random.default_rng(7)
    k = 4
    Wb, h1 = tie_case(rng, k=k)
    E, H = Wb.shape
    M = h1.shape[0]
    d, ref = oracle_router(Wb, h1, k)
    # the construction really ties: duplicated rows give equal oracle logits,
    # and the boundary pair straddles rank k
    assert np.all(ref["logits"][:, 2] == ref["logits"][:, 13])
    assert np.all(ref["logits"][:, 6] == ref["logits"][:, 11])
    for t in range(M):
        assert list(ref["idx"][t][:2]) == [2, 13] and ref["idx"][t][k - 1] == 6
        assert 11 not in ref["idx"][t]
    idx = torch.full((M, k), -1, dtype=torch.int32, device="cuda")
    gates = torch.zeros((M, k), dtype=torch.float32, device="cuda")
    kd.router_topk_static(torch_bf16(Wb), None, kd.KD_WBF16, None,
                          torch.from_numpy(h1).cuda(), M, H, E, k, idx, gates)
    torch.cuda.synchronize()
    gi, gg = idx.cpu().numpy(), gates.cpu().numpy()
    assert np.array_equal(gi, ref["idx"]), (gi, ref["idx"])
    assert np.abs(gg - ref["gates"]).max() < 1e-5
