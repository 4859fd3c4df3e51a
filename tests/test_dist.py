"""The multi-rank host logic of bench.py on CPU (gloo, world size 2).

The path is independent per (batch, head): bench.py's default multi-GPU mode
splits the heads of one problem over the ranks with no exchange step, so the
only cross-rank operations are the max-over-ranks reduction of the timed
region and the sum of the ranks' selected pairs; whole-job throughput counts
every rank's work.  The head split is checked here with the oracle on each
rank's heads: gathered, the shards' selections and outputs equal the
unsharded problem's.
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


SHARD_W = dict(name="shard5", heads=5, head_dim=64, text_len=40, num_frames=2, latent_h=8,
               latent_w=12, q_block=64, k_block=64, top_p=0.75, seed=41, kind="tiny")


def _shard_worker(rank, world, port, q):
    import dataclasses
    import datetime
    import numpy as np
    import torch.distributed as dist
    import bench
    import oracle
    from block_sparse_attention_45_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.custom(**SHARD_W)
        h0, h1 = bench.head_shard(w.heads, world, rank)
        ws = dataclasses.replace(w, heads=h1 - h0)
        x = synth.generate(ws, heads=range(h0, h1))
        tp = [w.top_p] * (h1 - h0)
        sel = oracle.select(ws.layout(), x["q"], x["k"], tp, w.flags)
        out, lse = oracle.attention(ws.layout(), x["q"], x["k"], x["v"], sel["mask"])
        pairs = bench.sum_over_ranks(int(sel["kv_count"].sum()))
        mine = dict(h0=h0, h1=h1, probs=sel["probs"], mask=sel["mask"], entropy=sel["entropy"],
                    kv_count=sel["kv_count"], out=out, lse=lse)
        got = [None] * world
        dist.all_gather_object(got, mine)
        q.put((rank, got if rank == 0 else None, pairs))
    finally:
        dist.destroy_process_group()


def test_head_shards_equal_the_whole_problem():
    import numpy as np
    import oracle
    from block_sparse_attention_45_b200 import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda r: r[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    shards = res[0][1]
    assert [(s["h0"], s["h1"]) for s in shards] == [(0, 2), (2, 5)]
    w = synth.custom(**SHARD_W)
    x = synth.generate(w)
    whole = oracle.select(w.layout(), x["q"], x["k"], [w.top_p] * w.heads, w.flags)
    out, lse = oracle.attention(w.layout(), x["q"], x["k"], x["v"], whole["mask"])
    cat = lambda key, ax=1: np.concatenate([s[key] for s in shards], axis=ax)  # noqa: E731
    for key in ("probs", "mask", "entropy", "kv_count"):     # [B, H, ...]
        assert np.array_equal(cat(key), whole[key]), key
    # attention rows come in (b, h, i) order; with one batch entry the shards follow each other
    assert np.array_equal(cat("out", 0), out) and np.array_equal(cat("lse", 0), lse)
    assert res[0][2] == res[1][2] == int(whole["kv_count"].sum())


def test_head_shard_covers_every_head_once():
    import bench
    for heads in (1, 5, 24, 40):
        for world in (1, 2, 3, 8):
            got = [h for r in range(world) for h in range(*bench.head_shard(heads, world, r))]
            assert got == list(range(heads))
            sizes = [bench.head_shard(heads, world, r)[1] - bench.head_shard(heads, world, r)[0]
                     for r in range(world)]
            assert max(sizes) - min(sizes) <= 1
