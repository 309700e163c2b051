"""World-size-2 checks of the benchmark's multi-rank plumbing on CPU (gloo): rendezvous, barrier,
max-over-ranks timing and the weak-scaling aggregate.  The data path itself has no collective:
every rank runs its own copy of the problem."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(0.5 + rank, world, torch.device("cpu"))
        units = bench.aggregate_weak(10.0, world)
        out[rank] = (t, units)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (1.5, 20.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    import bench

    class A:
        workload = "tiny"
        steps = 1
        warmup = 0

    assert bench.run_reference(A(), 2, 1) is None
