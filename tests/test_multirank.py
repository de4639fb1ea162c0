"""The multi-rank host logic of bench.py on CPU: two gloo ranks (127.0.0.1).

Each rank draws its own batch (weak scaling, no collective on the data path); the job's
time is the max over ranks; the job's rate counts the units of all ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import bench
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seed = bench.rank_seed(rank)
        batch = synth.kv_prefill_batch(2, 8, 128, seed=seed)
        times = [10.0 + rank, 3.0 * (rank + 1)]
        mx = bench.max_over_ranks(times, dist, torch.device("cpu"))
        dist.barrier()
        q.put((rank, seed, batch.sum(dtype=np.uint64).item(), mx, bench.job_rate(1000, world, mx[0])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, h0, m0, v0), (r1, s1, h1, m1, v1) = res
    assert s0 != s1 and h0 != h1                  # independent batches per rank
    assert m0 == m1 == [11.0, 6.0]                 # max over ranks, identical on every rank
    assert v0 == v1 == pytest.approx(2 * 1000 / (11.0 / 1e3) / 1e6)
