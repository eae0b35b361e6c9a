"""Pins of the CPU oracle against facts fixed by the mathematics, not by the
oracle itself: a hand-computed layer, closed forms, brute-force dense
evaluation, invariants of the gating, and library decoders.

The layer is the chain of the pages (wireai.ir "vLLM Blackwell Kimi decode",
section "4 key changes"; bigchange.ai "where the time went"): fused QKV
projection, o-proj + residual, router top-k with a softmax renormalised over the
selection, shared + routed SwiGLU experts, weighted combine.
"""
import math

import numpy as np
import pytest
import torch

import kdgen
import oracle
from kdgen import Dims, TINY

KIND = {"wqkv": 1, "wo": 2, "wr": 3, "wg": 4, "wu": 5, "wd": 6}


def tiny_inputs(dims=TINY, M=1, seed=0, rho=0.0):
    x = kdgen.bf16_bits_to_f32(kdgen.activations(seed, 0, kdgen.HIDDEN_IN, M, dims.hidden, rho))
    a = kdgen.bf16_bits_to_f32(kdgen.activations(seed, 0, kdgen.ATTN_OUT, M, dims.attn, rho))
    return x.astype(np.float64), a.astype(np.float64)


def explicit_weights(dims, wdtype=0, seed=0):
    """The generated weights as explicit fp64 arrays (shared expert first)."""
    def mat(kind, e=-1):
        R = {1: dims.nqkv, 2: dims.hidden, 3: dims.n_experts, 4: dims.inter, 5: dims.inter,
             6: dims.hidden}[kind]
        return oracle.weight_rows(dims, kind, e, 0, R, wdtype=wdtype, seed=seed)
    ex = ([-1] if dims.n_shared else []) + list(range(dims.n_experts))
    return {
        "wqkv": mat(1), "wo": mat(2), "wr": mat(3),
        "wg": np.stack([mat(4, e) for e in ex]),
        "wu": np.stack([mat(5, e) for e in ex]),
        "wd": np.stack([mat(6, e) for e in ex]),
    }


def silu(z):
    return z / (1.0 + math.exp(-z))


# ------------------------------------------------------------------ decoders

def test_bf16_decoder_matches_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2**16, 4000).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    ours = np.array([oracle.bf16_value(int(b)) for b in bits])
    assert np.array_equal(ours, ref)


def test_e4m3_decoder_matches_torch_all_codes():
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ours = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2
    assert np.array_equal(ours[~nan], ref[~nan])


def test_weight_rows_match_generator():
    # the oracle's row indexing (row * K + col, per matrix kind / expert slot)
    # against the generator's whole-matrix fill
    d = TINY
    for kind, e, R, K in [(1, -1, d.nqkv, d.hidden), (2, -1, d.hidden, d.attn),
                          (3, -1, d.n_experts, d.hidden), (4, 3, d.inter, d.hidden),
                          (5, -1, d.inter, d.hidden), (6, 7, d.hidden, d.inter)]:
        slot = 0 if kind <= 3 or e < 0 else e + 1
        ref = kdgen.bf16_bits_to_f32(kdgen.weight_bf16(0, 0, kind, slot, R, K)).astype(np.float64)
        assert np.array_equal(oracle.weight_rows(d, kind, e, 0, R), ref)
        assert np.array_equal(oracle.weight_rows(d, kind, e, 5, 3), ref[5:8])


def test_fp8_weight_rows_match_torch_decoding():
    d = TINY
    for kind, e, R, K in [(1, -1, d.nqkv, d.hidden), (3, -1, d.n_experts, d.hidden),
                          (6, 2, d.hidden, d.inter)]:
        slot = 0 if kind <= 3 else e + 1
        codes, scales = kdgen.weight_fp8(0, 0, kind, slot, R, K)
        deq = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
        sc = np.repeat(np.repeat(scales.astype(np.float64), 128, 0), 128, 1)[:R, :K]
        assert np.array_equal(oracle.weight_rows(d, kind, e, 0, R, wdtype=1), deq * sc)
        assert np.array_equal(oracle.weight_rows(d, kind, e, 130 if R > 131 else 1, 2, wdtype=1),
                              (deq * sc)[130 if R > 131 else 1:][:2])


# ------------------------------------------------------------- hand computed

MICRO = Dims(hidden=2, q_heads=1, kv_heads=0, head_dim=2, n_experts=2, top_k=1, n_shared=1, inter=1)


def micro_weights():
    return {
        "wqkv": np.array([[1.0, 2.0], [3.0, 4.0]]),
        "wo": np.array([[0.5, 0.0], [0.0, 0.5]]),
        "wr": np.array([[1.0, 0.0], [0.0, 1.0]]),
        # shared, expert 0, expert 1
        "wg": np.array([[[1.0, 0.0]], [[0.0, 1.0]], [[5.0, 5.0]]]),
        "wu": np.array([[[0.0, 1.0]], [[1.0, 1.0]], [[5.0, 5.0]]]),
        "wd": np.array([[[1.0], [0.0]], [[0.0], [2.0]], [[9.0], [9.0]]]),
    }


def test_hand_computed_layer():
    # x = (1, -1), a = (2, 4):
    #   qkv = (1-2, 3-4) = (-1, -1);  h1 = x + (1, 2) = (2, 1)
    #   logits = (2, 1) -> top-1 = expert 0, gate 1
    #   shared: silu(2) * 1 on row 0  -> s = (silu 2, 0)
    #   expert 0: gate 1, up 3 -> act = 3 silu(1); down (0, 2) -> (0, 6 silu 1)
    r = oracle.layer(MICRO, np.array([[1.0, -1.0]]), np.array([[2.0, 4.0]]), weights=micro_weights())
    assert np.array_equal(r["qkv"], [[-1.0, -1.0]])
    assert np.array_equal(r["h1"], [[2.0, 1.0]])
    assert np.array_equal(r["logits"], [[2.0, 1.0]])
    assert list(r["idx"][0]) == [0] and r["gates"][0, 0] == 1.0
    assert np.allclose(r["out"], [[2.0 + silu(2.0), 1.0 + 6.0 * silu(1.0)]], rtol=1e-15, atol=0)
    assert abs(r["out"][0, 0] - 3.7615941559557646) < 1e-14
    assert abs(r["out"][0, 1] - 5.386351471780029) < 1e-14


def test_hand_computed_selection_flips_with_bias():
    # bias (0, 5) makes expert 1 win: act = silu(5 * 3) * 15, down (9, 9)
    r = oracle.layer(MICRO, np.array([[1.0, -1.0]]), np.array([[2.0, 4.0]]), weights=micro_weights(),
                     bias=np.array([0.0, 5.0]))
    assert list(r["idx"][0]) == [1]
    assert np.array_equal(r["logits"], [[2.0, 6.0]])
    v = 9.0 * silu(15.0) * 15.0
    assert np.allclose(r["out"], [[2.0 + silu(2.0) + v, 1.0 + v]], rtol=1e-15, atol=0)


# ------------------------------------------------------------- closed forms

def test_zero_projections_return_input():
    d = TINY
    w = explicit_weights(d)
    w["wo"][:] = 0.0
    w["wd"][:] = 0.0
    x, a = tiny_inputs(d, M=3)
    r = oracle.layer(d, x, a, weights=w)
    assert np.array_equal(r["h1"], x)
    assert np.array_equal(r["out"], x)


def test_one_hot_inputs_pick_columns():
    d = TINY
    w = explicit_weights(d)
    for c in (0, 17, d.hidden - 1):
        x = np.zeros((1, d.hidden)); x[0, c] = 1.0
        a = np.zeros((1, d.attn)); a[0, (3 * c) % d.attn] = 1.0
        r = oracle.layer(d, x, a, weights=w)
        assert np.array_equal(r["qkv"][0], w["wqkv"][:, c])
        h1 = w["wo"][:, (3 * c) % d.attn].copy(); h1[c] += 1.0
        assert np.array_equal(r["h1"][0], h1)


def test_top1_gate_is_one_and_topE_is_dense_softmax():
    base = TINY
    x, a = tiny_inputs(base, M=4)
    for k in (1, base.n_experts):
        d = Dims(**{**base.__dict__, "top_k": k})
        r = oracle.layer(d, x, a)
        if k == 1:
            assert np.all(r["gates"] == 1.0)
            assert np.array_equal(r["idx"][:, 0], np.argmax(r["logits"], axis=1))
        else:
            l = r["logits"]
            sm = np.exp(l - l.max(1, keepdims=True)); sm /= sm.sum(1, keepdims=True)
            got = np.zeros_like(sm)
            for t in range(4):
                got[t, r["idx"][t]] = r["gates"][t]
            assert np.allclose(got, sm, rtol=1e-14, atol=1e-16)


def test_gate_ratios_are_exp_of_logit_gaps():
    x, a = tiny_inputs(TINY, M=5)
    r = oracle.layer(TINY, x, a)
    for t in range(5):
        i, j = r["idx"][t]
        l = r["logits"][t]
        assert abs(r["gates"][t, 0] / r["gates"][t, 1] - math.exp(l[i] - l[j])) < 1e-13
        assert abs(r["gates"][t].sum() - 1.0) < 1e-15
        assert np.all(r["gates"][t] > 0)


# ------------------------------------------------------------- brute force

def dense_reference(d, w, x, a, bias=None):
    """Brute force: every expert on every token, weighted by the selection mask
    times the softmax restricted to the mask; the selection is found by
    scanning all size-k subsets for the largest logit sum."""
    import itertools
    M = x.shape[0]
    h1 = x + a @ w["wo"].T
    lg = h1 @ w["wr"].T + (0 if bias is None else bias)
    out = h1.copy()
    ex = w["wg"].shape[0]
    F = []
    for e in range(ex):
        g = h1 @ w["wg"][e].T
        u = h1 @ w["wu"][e].T
        F.append((g / (1 + np.exp(-g)) * u) @ w["wd"][e].T)
    if d.n_shared:
        out += F[0]
    R = F[d.n_shared:]
    for t in range(M):
        best = max(itertools.combinations(range(d.n_experts), d.top_k),
                   key=lambda s: (sum(lg[t, list(s)]), [-i for i in s]))
        mask = np.zeros(d.n_experts, bool); mask[list(best)] = True
        p = np.where(mask, np.exp(lg[t] - lg[t, mask].max()), 0.0)
        p /= p.sum()
        for e in range(d.n_experts):
            out[t] += p[e] * R[e][t]
    return x @ w["wqkv"].T, h1, lg, out


@pytest.mark.parametrize("k", [1, 2, 3])
def test_sparse_equals_dense_brute_force(k):
    d = Dims(**{**TINY.__dict__, "top_k": k})
    w = explicit_weights(d)
    x, a = tiny_inputs(d, M=6)
    bias = kdgen.zipf_bias(d.n_experts, 1.1).astype(np.float64)
    r = oracle.layer(d, x, a, weights=w, bias=bias)
    qkv, h1, lg, out = dense_reference(d, w, x, a, bias)
    assert np.allclose(r["qkv"], qkv, rtol=1e-12, atol=1e-13)
    assert np.allclose(r["h1"], h1, rtol=1e-12, atol=1e-13)
    assert np.allclose(r["logits"], lg, rtol=1e-12, atol=1e-13)
    rel = np.abs(r["out"] - out).max() / np.sqrt((out ** 2).mean())
    assert rel < 1e-12


def test_seeded_equals_explicit_generated_weights():
    d = TINY
    x, a = tiny_inputs(d, M=3)
    for wd in (0, 1):
        r1 = oracle.layer(d, x, a, wdtype=wd)
        r2 = oracle.layer(d, x, a, weights=explicit_weights(d, wdtype=wd))
        for k in ("qkv", "h1", "logits", "gates", "out"):
            assert np.array_equal(r1[k], r2[k]), k


# ------------------------------------------------------------- invariants

def test_only_selected_experts_contribute():
    d = TINY
    w = explicit_weights(d)
    x, a = tiny_inputs(d, M=1)
    r = oracle.layer(d, x, a, weights=w)
    sel = set(r["idx"][0].tolist())
    w2 = {k: v.copy() for k, v in w.items()}
    rng = np.random.default_rng(5)
    for e in range(d.n_experts):
        if e not in sel:
            for k in ("wg", "wu", "wd"):
                w2[k][d.n_shared + e] = rng.standard_normal(w2[k][d.n_shared + e].shape)
    r2 = oracle.layer(d, x, a, weights=w2)
    assert np.array_equal(r["out"], r2["out"])
    # changing a selected expert does change the result
    e = r["idx"][0, 0]
    w2["wd"][d.n_shared + e] *= 2.0
    assert not np.array_equal(oracle.layer(d, x, a, weights=w2)["out"], r["out"])


def test_rows_are_independent():
    d = TINY
    x, a = tiny_inputs(d, M=5, rho=0.9)
    r = oracle.layer(d, x, a)
    for t in range(5):
        rt = oracle.layer(d, x[t:t + 1], a[t:t + 1])
        for k in ("qkv", "h1", "logits", "gates", "out"):
            assert np.array_equal(r[k][t], rt[k][0]), k
        assert np.array_equal(r["idx"][t], rt["idx"][0])


@pytest.mark.parametrize("ks", [2, 7, 56])
def test_split_k_agrees(ks):
    d = TINY
    x, a = tiny_inputs(d, M=2)
    r1 = oracle.layer(d, x, a, ksplit=1)
    r2 = oracle.layer(d, x, a, ksplit=ks)
    assert np.array_equal(r1["idx"], r2["idx"])
    for k in ("qkv", "h1", "logits", "out"):
        rel = np.abs(r1[k] - r2[k]).max() / np.sqrt((r1[k] ** 2).mean())
        assert rel < 1e-12


def test_threads_do_not_change_results():
    d = TINY
    x, a = tiny_inputs(d, M=4)
    r1 = oracle.layer(d, x, a, nthreads=1)
    r2 = oracle.layer(d, x, a, nthreads=4)
    for k in ("qkv", "h1", "logits", "gates", "out"):
        assert np.array_equal(r1[k], r2[k])


def test_exact_tie_takes_lower_index():
    d = Dims(hidden=2, q_heads=1, kv_heads=0, head_dim=2, n_experts=4, top_k=2, n_shared=0, inter=1)
    w = {
        "wqkv": np.eye(2), "wo": np.zeros((2, 2)),
        "wr": np.array([[0.0, 1.0], [1.0, 0.0], [1.0, 0.0], [1.0, 0.0]]),
        "wg": np.ones((4, 1, 2)), "wu": np.ones((4, 1, 2)), "wd": np.ones((4, 2, 1)),
    }
    r = oracle.layer(d, np.array([[1.0, 0.0]]), np.zeros((1, 2)), weights=w)
    # logits (0, 1, 1, 1): the two selected are experts 1 and 2
    assert list(r["idx"][0]) == [1, 2]
    assert np.array_equal(r["gates"][0], [0.5, 0.5])


def test_bias_shift_invariance_and_expert_permutation():
    d = TINY
    w = explicit_weights(d)
    x, a = tiny_inputs(d, M=3)
    b = kdgen.zipf_bias(d.n_experts, 1.1).astype(np.float64)
    r = oracle.layer(d, x, a, weights=w, bias=b)
    r2 = oracle.layer(d, x, a, weights=w, bias=b + 3.0)
    assert np.array_equal(r["idx"], r2["idx"])
    assert np.allclose(r["gates"], r2["gates"], rtol=1e-14)
    # relabel routed experts by a permutation: selection relabels, output stays
    perm = np.array([5, 2, 7, 0, 1, 6, 3, 4])  # new expert j = old expert perm[j]
    w3 = dict(w)
    w3["wr"] = w["wr"][perm]
    for k in ("wg", "wu", "wd"):
        w3[k] = np.concatenate([w[k][:1], w[k][1:][perm]])
    r3 = oracle.layer(d, x, a, weights=w3, bias=b[perm])
    inv = np.argsort(perm)
    for t in range(3):
        assert sorted(perm[r3["idx"][t]].tolist()) == sorted(r["idx"][t].tolist())
    assert np.allclose(r3["out"], r["out"], rtol=1e-13, atol=1e-13)


def test_forced_selection_recomputes_gates():
    d = TINY
    x, a = tiny_inputs(d, M=2)
    r = oracle.layer(d, x, a)
    forced = np.array([[0, 1], [6, 3]], np.int32)
    rf = oracle.layer(d, x, a, forced_idx=forced)
    assert np.array_equal(rf["idx"], forced)
    for t in range(2):
        l = r["logits"][t, forced[t]]
        p = np.exp(l - l.max()); p /= p.sum()
        assert np.allclose(rf["gates"][t], p, rtol=1e-14)
    assert np.array_equal(rf["h1"], r["h1"])


def test_golden_tiny_regression():
    """Oracle output on the tiny workload, written by tests/golden/make_golden.py."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_seed0.txt")
    lines = [l for l in open(path) if not l.startswith("#")]
    vals = {}
    for l in lines:
        k, rest = l.split(":", 1)
        vals[k.strip()] = np.array([float(v) for v in rest.split()])
    w = kdgen.WORKLOADS["tiny"]
    x = kdgen.bf16_bits_to_f32(w.hidden_in()).astype(np.float64)
    a = kdgen.bf16_bits_to_f32(w.attn_out()).astype(np.float64)
    r = oracle.layer(w.dims, x, a)
    assert np.array_equal(r["idx"][0], vals["idx"].astype(int))
    for k in ("gates", "out"):
        assert np.allclose(r[k][0], vals[k], rtol=1e-12, atol=1e-14), k


# ------------------------------------------------------------- gating variants

TRI = Dims(hidden=2, q_heads=1, kv_heads=0, head_dim=2, n_experts=3, top_k=2, n_shared=1, inter=1)


def tri_weights(shared_down=1.0):
    # Wo = 0 so h1 = x = (1, 1); router logits (3, 2, 1); every expert's
    # SwiGLU value is silu(1) * 1 on row 0, times its own down column
    return {
        "wqkv": np.zeros((2, 2)), "wo": np.zeros((2, 2)),
        "wr": np.array([[3.0, 0.0], [2.0, 0.0], [1.0, 0.0]]),
        "wg": np.array([[[1.0, 0.0]]] * 4), "wu": np.array([[[1.0, 0.0]]] * 4),
        "wd": np.array([[[shared_down], [0.0]], [[1.0], [0.0]], [[0.0], [1.0]], [[1.0], [1.0]]]),
    }


def test_selection_only_bias_hand_computed():
    # bias (0, 0, 2.5): keys (3, 2, 3.5) select experts 2 then 0.  Gates over
    # the selection: biased logits (3.5, 3) in the plain reading, unbiased
    # (1, 3) with the selection-only bias.
    x, a = np.array([[1.0, 1.0]]), np.zeros((1, 2))
    b = np.array([0.0, 0.0, 2.5])
    plain = oracle.layer(TRI, x, a, weights=tri_weights(), bias=b)
    sel = oracle.layer(TRI, x, a, weights=tri_weights(), bias=b, bias_select_only=True)
    assert list(plain["idx"][0]) == [2, 0] and list(sel["idx"][0]) == [2, 0]
    assert np.allclose(plain["gates"][0], [1 / (1 + math.exp(-0.5)), 1 / (1 + math.exp(0.5))],
                       rtol=1e-15)
    assert np.allclose(sel["gates"][0], [1 / (1 + math.exp(2.0)), 1 / (1 + math.exp(-2.0))],
                       rtol=1e-15)
    assert np.array_equal(sel["logits"][0], [3.0, 2.0, 1.0])      # unbiased
    assert np.array_equal(plain["logits"][0], [3.0, 2.0, 3.5])    # biased
    # out = h1 + silu(1) (shared down (1, 0)) + sum_j g_j silu(1) down_{e_j}
    s1 = silu(1.0)
    g2, g0 = sel["gates"][0]
    want = np.array([1 + s1 + g2 * s1 * 1.0 + g0 * s1 * 1.0, 1 + g2 * s1 * 1.0 + g0 * 0.0])
    assert np.allclose(sel["out"][0], want, rtol=1e-15)


def test_routed_scale_multiplies_the_routed_sum():
    x, a = tiny_inputs(M=3)
    base = oracle.layer(TINY, x, a, want_qkv=False)
    for s in (0.5, 2.5):
        r = oracle.layer(TINY, x, a, want_qkv=False, routed_scale=s)
        assert np.array_equal(r["idx"], base["idx"])
        # shared part: the layer with the routed sum scaled by 0 is h1 + shared
        sh = oracle.layer(TINY, x, a, want_qkv=False, routed_scale=1e-300)["out"]
        assert np.allclose(r["out"] - sh, s * (base["out"] - sh), rtol=1e-12, atol=1e-13)


def test_selection_only_bias_equals_plain_without_bias():
    x, a = tiny_inputs(M=2)
    r0 = oracle.layer(TINY, x, a, want_qkv=False)
    r1 = oracle.layer(TINY, x, a, want_qkv=False, bias=np.zeros(TINY.n_experts),
                      bias_select_only=True)
    assert np.array_equal(r0["out"], r1["out"]) and np.array_equal(r0["idx"], r1["idx"])
