"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The attention path has no collective: each GPU runs its own independent
problems.  Only the timing crosses ranks: a barrier around the timed region
and the max over ranks of the measured times.  This checks that logic with
two CPU processes.
"""
import os
import socket

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
    # the bench's aggregation: each rank timed `steps` steps of its own
    # problems; value = units of all ranks / the slowest rank's time
    steps, units = 20, 5.0e11
    fwd_ms = [60.0, 75.0][rank]
    (max_ms,) = bench.reduce_max([fwd_ms], w)
    rate = bench.job_rate(units, steps, w, max_ms)
    out[rank] = torch.tensor(vals + [max_ms, rate])
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
        got = out[r].tolist()
        assert got[:3] == [2.0, 10.0, 0.5]
        assert got[3] == 75.0
        # 2 ranks x 20 steps x 5e11 units in 75 ms
        assert abs(got[4] - 2 * 20 * 5.0e11 / 0.075) <= 1e-6 * got[4]


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.reduce_max([1.0, 2.0], 1) == [1.0, 2.0]
    bench.barrier(1)


def test_launch_plan():
    import bench

    assert bench.launch_plan(1, {}) == "run"
    assert bench.launch_plan(8, {}) == "spawn"
    assert bench.launch_plan(4, {"WORLD_SIZE": "4"}) == "run"
    assert bench.launch_plan(8, {"WORLD_SIZE": "2"}).startswith("error")
    assert bench.launch_plan(0, {}).startswith("error")


def test_mismatched_world_size_is_refused():
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "8"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "WORLD_SIZE=2" in r.stderr
