"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): every rank codes
its own disjoint batch (weak scaling, no data-path collective) and timings are reduced
as the max over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        layers = bench.rank_layers(32, rank, world)
        mx = bench.max_over_ranks(1.0 + rank, world)
        sm = bench.sum_over_ranks(10.0 * (rank + 1), world)
        q.put((rank, layers, mx, sm))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_reduce():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    l0, l1 = res[0][1], res[1][1]
    assert len(l0) == len(l1) == 32 and not set(l0) & set(l1)
    assert all(r[2] == 2.0 for r in res)          # max over ranks
    assert all(r[3] == 30.0 for r in res)         # sum over ranks


def test_single_rank_is_identity():
    import bench
    assert bench.rank_layers(32, 0, 1) == list(range(32))
    assert bench.max_over_ranks(3.5, 1) == 3.5
