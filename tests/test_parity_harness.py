"""The comparison logic of the GPU parity tests, exercised on the CPU with
planted results: a near-tie the GPU resolved the other way is excused and
its row recomputed under the GPU's selection; a flipped selection that is
not a near tie, an output off by more than the tolerance, and an output off
by a dropped activation term all fail.  The "GPU" results here are made by
the oracle itself (with a forced selection or a planted error), so no GPU
is needed."""
import numpy as np
import pytest

import kdgen
import oracle
from kdgen import TINY
from kdtest import TIE_GAP, TOL, compare_layer

D = TINY


def _inputs(M=3):
    x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, D.hidden, 0.2)
    a = kdgen.activations(0, 0, kdgen.ATTN_OUT, M, D.attn, 0.2)
    return x, a


def _f64(bits):
    return kdgen.bf16_bits_to_f32(bits).astype(np.float64)


def _as_gpu(ref, M):
    """An oracle result dressed as a GPU result (bf16 outputs, fp32 debug)."""
    return {"out": kdgen.to_bf16_bits(ref["out"].astype(np.float32)),
            "qkv": kdgen.to_bf16_bits(ref["qkv"].astype(np.float32)),
            "h1": ref["h1"].astype(np.float32), "logits": ref["logits"].astype(np.float32),
            "idx": ref["idx"].copy(), "gates": ref["gates"].astype(np.float32),
            "counts": np.bincount(ref["idx"].ravel(), minlength=D.n_experts).astype(np.int32),
            "n_active": int(len(np.unique(ref["idx"])))}


def _near_tie_bias(x, a, t, gap):
    """A router bias that puts token t's k-th and (k+1)-th logits `gap` apart."""
    base = oracle.layer(D, _f64(x), _f64(a))
    lg = base["logits"][t]
    order = np.argsort(-lg, kind="stable")
    ek, ek1 = order[D.top_k - 1], order[D.top_k]
    bias = np.zeros(D.n_experts)
    bias[ek1] = lg[ek] - lg[ek1] - gap
    return bias, ek, ek1


def test_exact_result_passes():
    x, a = _inputs()
    ref = oracle.layer(D, _f64(x), _f64(a))
    r = compare_layer(D, _as_gpu(ref, 3), x, a, strict_raw=True)
    assert r["excused"] == [] and r["out"] == 0.0


def test_near_tie_is_excused_and_recomputed():
    x, a = _inputs()
    bias, ek, ek1 = _near_tie_bias(x, a, 1, 0.3 * TIE_GAP)
    ref = oracle.layer(D, _f64(x), _f64(a), bias=bias)
    assert ek in ref["idx"][1] and ek1 not in ref["idx"][1]
    # the "GPU" took the (k+1)-th expert for token 1
    forced = ref["idx"].copy()
    forced[1][list(forced[1]).index(ek)] = ek1
    flipped = oracle.layer(D, _f64(x), _f64(a), bias=bias, forced_idx=forced)
    r = compare_layer(D, _as_gpu(flipped, 3), x, a, bias=bias)
    assert r["excused"] == [1]
    assert r["out"] == 0.0   # compared with the oracle recomputed under the GPU's selection


def test_flip_without_near_tie_fails():
    x, a = _inputs()
    bias, ek, ek1 = _near_tie_bias(x, a, 1, 30 * TIE_GAP)
    ref = oracle.layer(D, _f64(x), _f64(a), bias=bias)
    forced = ref["idx"].copy()
    forced[1][list(forced[1]).index(ek)] = ek1
    flipped = oracle.layer(D, _f64(x), _f64(a), bias=bias, forced_idx=forced)
    with pytest.raises(AssertionError, match="not a near tie"):
        compare_layer(D, _as_gpu(flipped, 3), x, a, bias=bias)


@pytest.mark.parametrize("rel", [1.5 * TOL[0], 1e-2])
def test_planted_output_error_fails(rel):
    # one element off by `rel` rms: above the tolerance, or the size of the
    # error a dropped activation term leaves (caught by the tight bound)
    x, a = _inputs()
    ref = oracle.layer(D, _f64(x), _f64(a))
    g = _as_gpu(ref, 3)
    rms = np.sqrt(np.mean(ref["out"] ** 2))
    bad = ref["out"].copy()
    bad[2, 17] += rel * rms + abs(bad[2, 17]) * 2.0 ** -8
    g["out"] = kdgen.to_bf16_bits(bad.astype(np.float32))
    with pytest.raises(AssertionError):
        compare_layer(D, g, x, a)
