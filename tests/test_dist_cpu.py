"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): each rank draws
its own batch of the same shape, timings reduce with max and token counts with
sum, and no data-path collective is needed."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from paged_kv_cache_473_b200 import workloads as wl

        w = wl.WORKLOADS["tinyllama_1b"]
        b = wl.make_batch(w, seed=bench.rank_seed(w, rank), batch=3, max_len=200)
        t = bench.max_over_ranks(float(rank + 1) * 1.5, world)
        n = bench.sum_over_ranks(float(b.q.shape[0]), world)
        q.put((rank, t, n, float(b.q.float().sum()), tuple(b.q.shape)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions_and_independent_batches():
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
    (r0, t0, n0, s0, sh0), (r1, t1, n1, s1, sh1) = res
    assert t0 == t1 == 3.0  # max over ranks
    assert n0 == n1 == 6.0  # tokens summed over ranks
    assert sh0 == sh1 and s0 != s1  # same shape, different draws
