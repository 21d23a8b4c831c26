"""The multi-GPU path of bench.py is replicas only: independent sequences per
rank, no collective on the data path.  Its harness (barrier, max-reduction of
the step time, whole-job aggregation) is checked here with two gloo ranks on
the CPU."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        bench.barrier(world)
        # rank r pretends its step took 10 + r ms for 4096 tokens
        ms, value = bench.aggregate(4096, 10.0 + rank, world)
        bench.barrier(world)
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_replica_timing_takes_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, value in got:
        assert ms == pytest.approx(11.0)                  # max over ranks
        assert value == pytest.approx(2 * 4096 / 11.0e-3)  # all ranks' tokens / slowest time
