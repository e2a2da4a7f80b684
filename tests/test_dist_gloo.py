"""Multi-process (world size 2, gloo, CPU) checks of the multi-GPU logic.

The WKV problems shard into independent (b, h) units, so one problem splits
along the batch with a single exchange: the backward's du, summed over the
ranks' batches by one all-reduce of C floats.  The timing crosses ranks too:
the step time is the maximum over ranks and the throughput counts every rank's
tokens.
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


# ---------------------------------------------------------------- one problem split along the batch

def test_batch_range_covers_every_batch_once():
    from linear_attention_rnn_wkv6_b200.shard import batch_range
    for B in (0, 1, 5, 32, 33, 256):
        for world in (1, 2, 3, 4, 8):
            ranges = [batch_range(B, r, world) for r in range(world)]
            covered = [b for lo, hi in ranges for b in range(lo, hi)]
            assert covered == list(range(B))
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        batch_range(4, 2, 2)


def _shard_worker(rank, world, port, q):
    """Rank `rank` of a batch-split backward: its batches of one seeded problem, the
    oracle's du partial over them, summed over ranks with the same collective the
    benchmark uses (gloo here, NCCL on GPUs)."""
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from linear_attention_rnn_wkv6_b200 import synth
        from linear_attention_rnn_wkv6_b200.shard import allreduce_du, batch_range
        B, T, H = 5, 20, 2
        lo, hi = batch_range(B, rank, world)
        x = synth.make_wkv6(B, T, H, seed=77, with_dy=True, batches=(lo, hi))
        f = [x.as_f64(n) for n in ("r", "k", "v", "w")] + [x.u.astype(np.float64)]
        dr, dk, dv, dw, du = oracle.wkv6_bwd(*f, x.dy.astype(np.float64), H=H, bidirectional=True)
        t = torch.from_numpy(du.copy())
        allreduce_du(t)
        q.put((rank, lo, hi, t.numpy(), dr))
    finally:
        dist.destroy_process_group()


def test_two_rank_batch_split_du_allreduce():
    import numpy as np
    import oracle
    from linear_attention_rnn_wkv6_b200 import synth
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    # the whole problem on one process
    x = synth.make_wkv6(5, 20, 2, seed=77, with_dy=True)
    f = [x.as_f64(n) for n in ("r", "k", "v", "w")] + [x.u.astype(np.float64)]
    dr, dk, dv, dw, du = oracle.wkv6_bwd(*f, x.dy.astype(np.float64), H=2, bidirectional=True)
    assert [(lo, hi) for _, lo, hi, _, _ in res] == [(0, 3), (3, 5)]
    for rank, lo, hi, du_sum, dr_part in res:
        assert np.allclose(du_sum, du, rtol=1e-12, atol=1e-12)   # identical on every rank
        assert np.array_equal(dr_part, dr[lo:hi])                # per-batch gradients need no exchange
