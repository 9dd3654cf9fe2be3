"""The benchmark's multi-rank host logic on CPU with gloo, world size 2: every rank runs an
independent replica, the barrier holds, and the reported time is the max over ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    d = bench.Dist(world, backend="gloo")
    d.barrier()
    ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
    m = d.max(ms)
    out[rank] = (d.world, d.rank, m, bench.job_throughput(d.world, 100, 1e6, m))
    d.barrier()
    d.close()


def test_two_ranks_max_over_ranks():
    ctx = mp.get_context("spawn")
    port = _free_port()
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0][2] == out[1][2] == 15.0           # both see the slower rank's time
    assert out[0][3] == pytest.approx(2 * 100 * 1e6 / 15e-3)
    assert {out[0][1], out[1][1]} == {0, 1} and out[0][0] == 2


def test_single_rank_is_identity():
    os.environ.pop("WORLD_SIZE", None)
    d = bench.Dist(1, backend="gloo")
    assert d.world == 1 and d.max(3.5) == 3.5
