"""The bench's multi-rank plumbing on CPU: two gloo ranks (one process per
rank, as under torchrun), the timing barrier, the max over ranks and the
whole-job metric, and the reference arm's rank-0-only rule."""
import contextlib
import io
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(dist, 0)
        m = bench.max_over_ranks(dist, 1.5 + rank)       # rank r took 1.5 + r ms
        q.put((rank, m, bench.job_us_per_layer(m, world)))
        bench.barrier(dist, 0)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    # every rank sees the slowest rank's time; the job processed 2 layers in it
    assert [g[1] for g in got] == [2.5, 2.5]
    assert all(g[2] == pytest.approx(2.5 * 1e3 / 2) for g in got)


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class A:
        workload, steps, warmup = "tiny", 1, 3

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(A())
    assert buf.getvalue() == ""
