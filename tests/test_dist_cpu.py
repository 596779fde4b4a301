"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The attention path has no collective: each GPU runs its own independent
problems.  Only the timing crosses ranks: a barrier around the timed region
and the max over ranks of the measured times.  This checks that logic with
two CPU processes.
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    r, w, _ = bench.dist_setup(world)
    assert (r, w) == (rank, world)
    bench.barrier(w)
    vals = bench.reduce_max([float(rank + 1), 10.0 - rank, 0.5 * rank], w)
    out[rank] = torch.tensor(vals)
    bench.barrier(w)
    dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        assert out[r].tolist() == [2.0, 10.0, 0.5]


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.reduce_max([1.0, 2.0], 1) == [1.0, 2.0]
    bench.barrier(1)
