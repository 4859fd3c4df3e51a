"""The multi-rank host logic of bench.py on CPU (gloo, world size 2).

Every rank runs its own problem (the path shards by head with no exchange
step), so the only cross-rank operation is the max-over-ranks reduction of
the timed region; whole-job throughput counts every rank's work.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        m = bench.max_over_ranks(ms)
        q.put((rank, m, bench.job_tflops(1e12, world, m)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, tf in res:
        assert m == 15.0                       # every rank sees the slowest rank's time
        assert abs(tf - 2 * 1e12 / 15e-3 / 1e12) < 1e-9


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_tflops(2e12, 1, 1.0) == pytest.approx(2000.0)
