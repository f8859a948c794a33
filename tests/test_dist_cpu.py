"""bench.py's multi-rank plumbing on two CPU processes (gloo): the same barrier, max / sum
reductions and weak-scaling aggregate that the NCCL ranks use on GPUs."""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import mla_inputs as mi
    d = bench.Dist(world, backend="gloo")
    d.init(torch)
    d.barrier(torch)
    res = {
        "max": d.reduce(torch, rank + 1.0, "max"),
        "sum": d.reduce(torch, rank + 1.0, "sum"),
        # rank r times steps of (r + 1) ms each and moves 1e9 bytes per step
        "agg": bench.aggregate(d, torch, [rank + 1.0] * 4, 1e9),
        "seed": bench.rank_config(mi.CONFIGS["v2"], rank).seed,
    }
    d.barrier(torch)
    d.close()
    out.put((rank, res))


def test_two_rank_reductions_and_weak_scaling_aggregate():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        r = results[rank]
        assert r["max"] == 2.0 and r["sum"] == 3.0
        ms_per_step, tbs = r["agg"]
        # slowest rank: 2 ms per step; work: 2 ranks x 1e9 bytes -> 1 TB/s for the job
        assert ms_per_step == pytest.approx(2.0)
        assert tbs == pytest.approx(1.0)
    assert results[0]["seed"] != results[1]["seed"]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(1, backend="gloo")
    assert not d.pg
    assert d.reduce(torch, 5.0, "sum") == 5.0
    assert bench.aggregate(d, torch, [2.0, 2.0], 4e9) == pytest.approx((2.0, 2.0))
