"""The N > 1 host path of bench.py on CPU: two gloo ranks, max-over-ranks
timing (the job's time is its slowest rank's), and the reference arm that
only rank 0 runs. Weak scaling: every rank runs its own replica of the
workload, so the only collective is this timing reduction."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        t = torch.tensor([10.0 * (rank + 1)], dtype=torch.float64)
        out[rank] = bench.max_over_ranks(t, world)
        # the reference arm: ranks other than 0 return at once without work
        if rank != 0:
            class A:  # minimal args
                steps, warmup, gpus = 1, 3, world
            out[world + rank] = bench.run_reference(A(), None)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == 20.0 and out[1] == 20.0
    assert out[world + 1] == 0


def test_max_over_ranks_single():
    assert bench.max_over_ranks(torch.tensor([3.5], dtype=torch.float64), 1) == 3.5
