"""Multi-rank host logic of the bench on CPU (gloo, world size 2).

The path has no data-path collective: every rank runs an independent batch.
What the ranks share is the report: the slowest rank's time and the sum of the
work units. These tests run that reduction over a real two-process gloo group.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench

        ms = [0.5, 0.7][rank]
        e2e = [3.0, 2.0][rank]
        units = [1000, 3000][rank]
        results[rank] = bench.reduce_over_ranks(ms, e2e, units)
    finally:
        dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(results)
    for r in range(2):
        ms, e2e, units = res[r]
        assert ms == 0.7 and e2e == 3.0 and units == 4000.0


def test_aggregate_is_units_over_slowest_rank():
    import bench

    value, t = bench.aggregate([0.5, 0.7], [1000, 3000])
    assert t == 0.7
    assert value == pytest.approx(4000 / 0.7e-3 / 1e6)


def test_reduce_without_group_is_identity():
    import bench

    assert bench.reduce_over_ranks(1.5, 2.5, 7) == (1.5, 2.5, 7.0)
