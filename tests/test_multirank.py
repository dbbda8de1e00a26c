"""Two gloo ranks on the CPU: the multi-GPU bookkeeping of bench.py.

Each rank owns its own batch of independent (b, h) problems; the only
cross-rank step is the max of the per-rank step time (outside the data
path).  The whole-job value is every rank's tokens over the slowest time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        ms_local = 10.0 + 5.0 * rank                     # rank 1 is slower
        value, ms = bench.aggregate(16384, ms_local, world, "cpu")
        out_q.put((rank, value, ms))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
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
    for rank, value, ms in res:
        assert ms == pytest.approx(15.0)
        assert value == pytest.approx(2 * 16384 / 15e-3)


def test_single_rank_is_local():
    import bench
    value, ms = bench.aggregate(100, 4.0, 1, "cpu")
    assert ms == 4.0 and value == pytest.approx(100 / 4e-3)
