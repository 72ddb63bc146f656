"""Host logic of bench.py's multi-rank path on CPU: two gloo ranks reduce
their step times to the maximum, and the whole-job value counts every rank's
bytes over that slowest time."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [1.0 + rank, 0.5 * (2 - rank), 0.25 + rank, 3.0 - rank]
        got = bench.max_over_ranks(mine, world)
        out[rank] = (got, bench.job_throughput(570425344, world, got[0]))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        ctx = mp.get_context("spawn")
        procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    expect = [2.0, 1.0, 1.25, 3.0]
    for r in range(world):
        got, value = res[r]
        assert got == pytest.approx(expect)
        # both ranks' bytes over the slowest step (2 ms)
        assert value == pytest.approx(2 * 570425344 / 2e-3 / 1e9)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
    assert bench.job_throughput(1000, 1, 1.0) == pytest.approx(1e-3)
