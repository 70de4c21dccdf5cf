"""N > 1 host logic of the bench on CPU: world-size-2 gloo ranks exercise the
barrier, the max-over-ranks timing and the weak-scaling aggregation that
bench.py uses under torchrun (where the backend is NCCL)."""

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


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        # rank r "took" 10 + 5 r ms for its steps
        t_max = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        value = bench.weak_scaling_value(154.6e9, 100, world, t_max)
        out[rank] = (t_max, value)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_and_weak_scaling():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    t0, v0 = out[0]
    t1, v1 = out[1]
    assert t0 == t1 == 15.0                       # the slowest rank's time, on every rank
    assert v0 == v1 == pytest.approx(154.6e9 * 100 * 2 / 15e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.weak_scaling_value(1e12, 1, 1, 1000.0) == pytest.approx(1.0)
