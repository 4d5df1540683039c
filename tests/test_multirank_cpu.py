"""The multi-rank logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Every rank runs its own batches (weak scaling, no collective on the data
path); the step time is the maximum over ranks and rank 0 reports
world x tokens / that time."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 1.0 + rank * 0.5  # rank 1 is the slower one
        dist.barrier()
        ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        value = bench.weak_scaling_value(5, world, ms)
        q.put((rank, ms, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_step_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, value in res:
        assert ms == pytest.approx(1.5)
        assert value == pytest.approx(2 * 5 / 1.5e-3)


def test_single_process_keeps_its_own_time():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, None, None) == 2.5
    assert bench.weak_scaling_value(1, 1, 1.0) == pytest.approx(1000.0)
