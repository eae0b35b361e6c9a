"""The tensor-parallel layer on CPU: gloo ranks (one process each, as under
torchrun) run moe_decode_layer_skinny_b200.tp.decode_tp with the oracle's
per-rank slices; the all-reduced / all-gathered result equals the unsharded
oracle layer to 1e-12 (fp64; only the order of additions differs), on every
rank, for 2 and 4 ranks."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(dims, M):
    import kdgen
    x = kdgen.bf16_bits_to_f32(kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, dims.hidden))
    a = kdgen.bf16_bits_to_f32(kdgen.activations(0, 0, kdgen.ATTN_OUT, M, dims.attn))
    return x.astype(np.float64), a.astype(np.float64)


def _rank_main(rank, world, port, q, dims_kw, M, bias_s):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import kdgen
    from moe_decode_layer_skinny_b200 import tp
    from tp_oracle_shard import OracleShard
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        dims = kdgen.Dims(**dims_kw)
        x, a = _inputs(dims, M)
        bias = kdgen.zipf_bias(dims.n_experts, bias_s).astype(np.float64) if bias_s else None
        shard = OracleShard(dims, rank, world, bias=bias)
        hidden = torch.from_numpy(x.copy())
        tp.decode_tp(shard, hidden, torch.from_numpy(a))
        q.put((rank, hidden.numpy(), shard.qkv, shard.idx))
    finally:
        dist.destroy_process_group()


def _run(world, dims, M, bias_s=0.0):
    import dataclasses

    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, dataclasses.asdict(dims), M,
                                                   bias_s)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=300) for _ in range(world)), key=lambda g: g[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("world", [2, 4])
def test_tp_ranks_sum_to_the_unsharded_layer(world):
    sys.path.insert(0, ROOT)
    import kdgen
    import oracle
    import oracle.tp as otp
    dims, M = kdgen.TINY, 3
    got = _run(world, dims, M)
    x, a = _inputs(dims, M)
    ref = oracle.layer(dims, x, a)
    scale = np.sqrt(np.mean(ref["out"] ** 2))
    for rank, out, qkv, idx in got:
        assert np.array_equal(idx, ref["idx"])
        assert np.abs(out - ref["out"]).max() / scale <= 1e-12
        # the rank's QKV rows are the unsharded projection's rows
        rows = otp.qkv_rows(dims, rank, world)
        assert np.abs(qkv - ref["qkv"][:, rows]).max() / np.sqrt(np.mean(ref["qkv"] ** 2)) <= 1e-12
    # every rank ends with the same hidden state
    for g in got[1:]:
        assert np.array_equal(g[1], got[0][1])


def test_tp_with_router_bias_and_replicated_kv_heads():
    """Four ranks over a layer with two kv heads (ranks share them) and a
    Zipf router bias (the selection depends on the gathered, biased logits)."""
    sys.path.insert(0, ROOT)
    import kdgen
    import oracle
    dims = kdgen.Dims(hidden=256, q_heads=8, kv_heads=2, head_dim=32, n_experts=16, top_k=4,
                      n_shared=1, inter=128)
    M = 4
    got = _run(4, dims, M, bias_s=1.1)
    x, a = _inputs(dims, M)
    ref = oracle.layer(dims, x, a, bias=kdgen.zipf_bias(dims.n_experts, 1.1).astype(np.float64))
    scale = np.sqrt(np.mean(ref["out"] ** 2))
    for _, out, _, idx in got:
        assert np.array_equal(idx, ref["idx"])
        assert np.abs(out - ref["out"]).max() / scale <= 1e-12


def test_shard_spans():
    sys.path.insert(0, ROOT)
    import kdgen
    import oracle.tp as otp
    K2 = kdgen.K2
    for R in (2, 4, 8):
        rows = np.concatenate([otp.qkv_rows(K2, r, R) for r in range(R)])
        # with kv heads divisible by R the ranks' QKV rows partition the output
        assert sorted(rows.tolist()) == list(range(K2.nqkv))
        assert [otp.span(K2.inter, r, R) for r in range(R)][-1][1] == K2.inter
    # fewer kv heads than ranks: ranks replicate the kv head their q heads read
    T = kdgen.TINY
    assert [otp.kv_span(T, r, 4) for r in range(4)] == [(0, 1)] * 4
    with pytest.raises(ValueError):
        otp.span(10, 0, 4)
