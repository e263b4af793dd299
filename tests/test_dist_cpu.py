"""The multi-process path of bench.py on CPU: two gloo ranks run independent replicas, the
barrier brackets the timed region and rank 0 reports the slowest rank's time, scaled by the
number of replicas (weak scaling, no collective on the data path)."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench  # noqa: E402
    try:
        w, r, _ = bench.dist_setup()
        assert (w, r) == (world, rank)
        bench.barrier(w)
        ms, value = bench.replica_throughput(10.0 + 5.0 * rank, w)  # rank 1 is slower
        q.put((rank, ms, value))
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_replicas_report_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 15.0                       # max over ranks, on every rank
        assert abs(value - 2 * 1000.0 / 15.0) < 1e-9


def test_single_process_needs_no_process_group():
    import bench
    ms, value = bench.replica_throughput(20.0, 1)
    assert ms == 20.0 and value == 50.0
