"""The tensor-parallel shards on one GPU: R shard layers (kd_config.tp_rank /
tp_size) run their kd_tp_* phases one after another on the same stream, with
the three exchanges done by torch in between (sum of the partial sums in rank
order, concatenation of the logit shards) -- the same calls a multi-GPU run
makes, with no kernel waiting for another rank's.  The result is compared with
the unsharded oracle layer: output and every shard's QKV rows within the
layer's tolerance, the selection exact (near-ties excused as for the whole
layer)."""
import numpy as np
import pytest

import kdgen
from kdtest import compare_layer, fetch, torch_bf16, torch_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kd(torch_cuda):
    import moe_decode_layer_skinny_b200 as kd
    kd.lib()
    return kd

SMALL = kdgen.Dims(hidden=512, q_heads=4, kv_heads=2, head_dim=128, n_experts=16, top_k=4,
                   n_shared=1, inter=512)
WIDE = kdgen.Dims(hidden=512, q_heads=4, kv_heads=2, head_dim=128, n_experts=256, top_k=8,
                  n_shared=1, inter=512)


def _shards(kd, dims, R, M, **kw):
    return [kd.Layer(kd.LayerSpec.from_dims(dims, max_tokens=M, tp_rank=r, tp_size=R, **kw), seed=0)
            for r in range(R)]


def run_tp(kd, layers, x_bits, a_bits):
    """One sharded decode step, the ranks one after another on this GPU."""
    import torch
    from moe_decode_layer_skinny_b200.tp import CudaShard
    M = x_bits.shape[0]
    shards = [CudaShard(L, M) for L in layers]
    hid = [torch_bf16(x_bits) for _ in shards]
    at = torch_bf16(a_bits)
    for sh, h in zip(shards, hid):
        sh.attn_partial(h, at)
    p = shards[0].p.clone()
    for sh in shards[1:]:
        p += sh.p
    for sh, h in zip(shards, hid):
        sh.router_shard(h, p)
    logits = torch.cat([sh.lshard for sh in shards], dim=1)
    for sh in shards:
        sh.moe_partial(logits)
    y = shards[0].y.clone()
    for sh in shards[1:]:
        y += sh.y
    for sh, h in zip(shards, hid):
        sh.combine(y, h)
    torch.cuda.synchronize()
    for L in layers:
        L.check()
    out = [torch_bits(h) for h in hid]
    return out, logits.cpu().numpy().astype(np.float64), p


def _qkv_of(kd, dims, layers, M):
    """Every shard's QKV rows scattered into the unsharded layout."""
    import oracle.tp as otp
    R = len(layers)
    full = np.zeros((M, dims.nqkv), np.uint16)
    for r, L in enumerate(layers):
        rows = otp.qkv_rows(dims, r, R)
        full[:, rows] = fetch(L.qkv_ptr(), (M, len(rows)), np.uint16)
    return full


# mma_min: 0 = the tensor-core kernels, 1000 = the CUDA-core kernels
@pytest.mark.parametrize("R,M,mma_min", [(2, 1, 1000), (4, 1, 1000), (2, 2, 1000), (2, 1, 0),
                                         (2, 8, 0), (4, 8, 0), (4, 16, 0)])
def test_tp_small(kd, R, M, mma_min):
    wdtype = 0
    x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, SMALL.hidden)
    a = kdgen.activations(0, 0, kdgen.ATTN_OUT, M, SMALL.attn)
    layers = _shards(kd, SMALL, R, M, wdtype=wdtype, mma_min_tokens=mma_min)
    try:
        out, logits, _ = run_tp(kd, layers, x, a)
        # every rank ends with the same hidden state
        for o in out[1:]:
            assert np.array_equal(o, out[0])
        L0 = layers[0]
        g = {"out": out[0], "qkv": _qkv_of(kd, SMALL, layers, M),
             "h1": fetch(L0.debug_ptr(kd.T_H1F), (M, SMALL.hidden), np.float32),
             "logits": logits,
             "idx": fetch(L0.debug_ptr(kd.T_IDX), (M, SMALL.top_k), np.int32),
             "gates": fetch(L0.debug_ptr(kd.T_GATES), (M, SMALL.top_k), np.float32)}
        for L in layers[1:]:   # the same selection on every shard
            assert np.array_equal(fetch(L.debug_ptr(kd.T_IDX), (M, SMALL.top_k), np.int32), g["idx"])
        r = compare_layer(SMALL, g, x, a, wdtype=wdtype)
        print("tp", R, M, r)
    finally:
        for L in layers:
            L.close()


@pytest.mark.parametrize("M", [1, 8])
def test_tp_fp8(kd, M):
    """FP8 shards (whole 128 x 128 scale blocks per shard: 256 experts over 2
    ranks)."""
    x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, WIDE.hidden)
    a = kdgen.activations(0, 0, kdgen.ATTN_OUT, M, WIDE.attn)
    layers = _shards(kd, WIDE, 2, M, wdtype=1)
    try:
        out, logits, _ = run_tp(kd, layers, x, a)
        L0 = layers[0]
        g = {"out": out[0], "qkv": _qkv_of(kd, WIDE, layers, M),
             "h1": fetch(L0.debug_ptr(kd.T_H1F), (M, WIDE.hidden), np.float32),
             "logits": logits,
             "idx": fetch(L0.debug_ptr(kd.T_IDX), (M, WIDE.top_k), np.int32),
             "gates": fetch(L0.debug_ptr(kd.T_GATES), (M, WIDE.top_k), np.float32)}
        r = compare_layer(WIDE, g, x, a, wdtype=1)
        print("tp fp8", M, r)
    finally:
        for L in layers:
            L.close()


def test_tp_k2(kd):
    """Full-size shards (H=7168, 256 experts, I=2048) over 2 ranks at M=1 and
    M=8: the same selection as the unsharded GPU layer, and every output row
    and QKV row against the oracle."""
    K2 = kdgen.K2
    for M in (1, 8):
        x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, K2.hidden)
        a = kdgen.activations(0, 0, kdgen.ATTN_OUT, M, K2.attn)
        whole = kd.Layer(kd.LayerSpec.from_dims(K2, max_tokens=M), seed=0)
        try:
            h = torch_bf16(x)
            whole.decode(h, torch_bf16(a), M)
            whole.check()
            idx_ref = fetch(whole.debug_ptr(kd.T_IDX), (M, K2.top_k), np.int32)
        finally:
            whole.close()
        layers = _shards(kd, K2, 2, M)
        try:
            out, logits, _ = run_tp(kd, layers, x, a)
            L0 = layers[0]
            g = {"out": out[0], "qkv": _qkv_of(kd, K2, layers, M),
                 "h1": fetch(L0.debug_ptr(kd.T_H1F), (M, K2.hidden), np.float32),
                 "logits": logits,
                 "idx": fetch(L0.debug_ptr(kd.T_IDX), (M, K2.top_k), np.int32),
                 "gates": fetch(L0.debug_ptr(kd.T_GATES), (M, K2.top_k), np.float32)}
        finally:
            for L in layers:
                L.close()
        assert np.array_equal(g["idx"], idx_ref)
        r = compare_layer(K2, g, x, a)
        print("tp k2", M, r)


def test_tp_config_errors(kd):
    """Shardings the layer refuses (KD_EINVAL), and the whole-layer call on a
    shard."""
    bad = [dict(tp_rank=2, tp_size=2), dict(tp_rank=1, tp_size=0), dict(tp_rank=0, tp_size=3)]
    for kw in bad:
        with pytest.raises(kd.KdError) as e:
            kd.Layer(kd.LayerSpec.from_dims(SMALL, max_tokens=4, **kw))
        assert e.value.code == kd.KD_EINVAL
    with pytest.raises(kd.KdError) as e:   # FP8 with a split 128-row scale block of the router
        kd.Layer(kd.LayerSpec.from_dims(SMALL, max_tokens=4, wdtype=1, tp_rank=0, tp_size=2))
    assert e.value.code == kd.KD_EINVAL
    L = kd.Layer(kd.LayerSpec.from_dims(SMALL, max_tokens=4, tp_rank=0, tp_size=2))
    try:
        import torch
        h = torch.zeros((1, SMALL.hidden), dtype=torch.bfloat16, device="cuda")
        a = torch.zeros((1, SMALL.attn), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(kd.KdError) as e:
            L.decode(h, a, 1)
        assert e.value.code == kd.KD_EINVAL
        with pytest.raises(kd.KdError) as e:
            L.tp_moe(5)
        assert e.value.code == kd.KD_ERANGE
    finally:
        L.close()
