"""Multi-process (world size 2, gloo, CPU) checks of the benchmark's rank logic.

The WKV problems shard into independent (b, h) units, so ranks never exchange
data; what crosses ranks is the timing: the step time is the maximum over
ranks and the throughput counts every rank's tokens.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, l = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    try:
        elapsed = 10.0 + 5.0 * rank           # rank 1 is the slow one
        mx = bench.max_over_ranks(elapsed, dist)
        tot = bench.sum_over_ranks(1000.0 * (rank + 1), dist)
        bench.barrier(dist)
        q.put((r, w, l, mx, tot))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for r, (rank, world, local, mx, tot) in enumerate(res):
        assert (rank, world, local) == (r, 2, r)
        assert mx == 15.0            # max over ranks, identical on every rank
        assert tot == 3000.0


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.sum_over_ranks(2.0, None) == 2.0


def test_reference_arm_only_rank0_prints(capsys, monkeypatch):
    import bench

    class A:
        steps, warmup = 1, 3
    bench.run_reference(A, rank=1, world=2)
    assert capsys.readouterr().out == ""
