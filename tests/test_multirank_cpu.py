"""The N > 1 path of the benchmark on CPU: two gloo ranks.

Channels are independent problems, so N GPUs run N independent batches with no
data-path collective (weak scaling); the only cross-rank steps are the barrier
and the max of the step times.  These tests run that host logic with the gloo
backend, and check that a rank that fails before the collective makes the
others fail fast (short process-group timeout) instead of hanging.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _init(rank, world, port, timeout_s=30):
    from datetime import timedelta

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=timedelta(seconds=timeout_s))


def _aggregate_worker(rank, world, port, q):
    import bench

    _init(rank, world, port)
    ms_local = [2.0, 3.5][rank]
    bench.barrier(world)
    ms, value = bench.aggregate(ms_local, world, 1000, torch.device("cpu"))
    q.put((rank, ms, value))
    dist.destroy_process_group()


def test_weak_scaling_aggregate_two_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_aggregate_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, ms, value in res:
        assert ms == 3.5                                # the slowest rank sets the step time
        assert value == pytest.approx(2 * 1000 / 3.5e-3)  # all ranks' units / that time


def _failing_worker(rank, world, port, q):
    _init(rank, world, port, timeout_s=5)
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()  # flush before dying
        os._exit(3)  # a rank that dies between steps, before the next collective
    try:
        t = torch.tensor([1.0])
        dist.all_reduce(t)
        q.put((rank, "completed"))
    except Exception as e:  # the surviving rank gets an error, not a hang
        q.put((rank, "error:" + type(e).__name__))


def test_dead_rank_surfaces_as_error():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_failing_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=60) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert res[1] == "left"
    assert res[0].startswith("error:")
