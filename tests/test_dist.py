"""The benchmark's multi-rank plumbing on CPU with two gloo ranks: every rank
runs its own copy of the workload (weak scaling, distinct seeds), timings are
reduced by max over ranks, and the whole-job value counts every rank's units
over the slowest rank's time."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        vals = bench.reduce_max([10.0 + rank, 5.0 - rank, 7.0])
        value = bench.weak_scaling_value(world, 3, 65536, vals[0])
        q.put((rank, vals, value, bench.rank_seed(0, rank)))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduction_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, vals, value, seed in res:
        assert vals == [11.0, 5.0, 7.0]               # max over ranks, on every rank
        assert value == pytest.approx(2 * 3 * 65536 / 11e-3)
    assert res[0][3] != res[1][3]                      # independent problems per rank


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.5]) == [1.5, 2.5]
    assert bench.weak_scaling_value(1, 2, 100, 1000.0) == pytest.approx(200.0)
