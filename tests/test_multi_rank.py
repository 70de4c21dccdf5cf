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


def _amax_exchange_rank(rank, world, port, q):
    import os
    import numpy as np
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads as W
        from fp8_delayed_scaling_quantize_b200.dist import AMAX_WORD, allreduce_amax
        # each rank's own micro-batch for three tensor roles (x, W, g)
        xs = [W.bf16_normal((4096,), std, 7000 + 10 * rank + i).float().numpy()
              for i, std in enumerate((0.02, 0.5, 1e-3))]
        local = [np.float32(oracle.amax(x)) for x in xs]
        rings = torch.zeros(3, 20, dtype=torch.int32)
        rings[:, AMAX_WORD] = torch.tensor([int(np.array([a], np.float32).view(np.int32)[0]) for a in local],
                                           dtype=torch.int32)
        rings[:, 3] = 12345 + rank  # another word of the ring: untouched by the exchange
        allreduce_amax(rings)
        group = rings[:, AMAX_WORD].numpy().view(np.float32).copy()
        # fold the exchanged amax into the oracle's ring of each role
        refs = [oracle.DelayedRing() for _ in range(3)]
        for r, a, fmt in zip(refs, group, (0, 0, 1)):
            r.fold(a, fmt)
        q.put((rank, [float(a) for a in local], [float(a) for a in group], int(rings[0, 3]),
               [float(r.scale) for r in refs]))
    finally:
        dist.destroy_process_group()


def test_dp_amax_exchange_two_ranks():
    """world size 2 on gloo: after the exchange both ranks hold, bit for bit,
    the larger of the two amax values of every role, so their rings (folded
    by the oracle here) publish the same next scales; no other ring word
    moves."""
    import multiprocessing as mp
    import socket
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    procs = [ctx.Process(target=_amax_exchange_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=60) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, loc0, grp0, w0, sc0), (_, loc1, grp1, w1, sc1) = out
    assert grp0 == grp1 == [max(a, b) for a, b in zip(loc0, loc1)]
    assert loc0 != loc1  # the ranks really had different data
    assert sc0 == sc1
    assert (w0, w1) == (12345, 12346)
