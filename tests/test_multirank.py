"""The N > 1 host path of bench.py on CPU ranks (gloo, world size 2).

Each rank runs the hot path on its own batch (independent sequences: no data
exchange), so the only collective is the timing reduction: the job's step
time is the slowest rank's, and the job's throughput counts every rank's
work over that time.
"""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms = [3.0, 5.0][rank]
        t = bench.max_over_ranks(ms, dist, "cpu")
        v = bench.job_throughput(world, 1e12, t)
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_timing_reduction_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, v in res:
        assert t == 5.0                       # the slowest rank
        assert v == pytest.approx(2 * 1e12 / 5e-3)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(4.0, None, "cpu") == 4.0
    assert bench.job_throughput(1, 2e12, 2.0) == pytest.approx(1e15)
