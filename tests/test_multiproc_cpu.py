"""Multi-process host logic of the benchmark, on CPU with the gloo backend (world size 2).

Every rank runs its own request (weak scaling): seeds differ per rank, the job time is
the slowest rank's device time, and the whole-job value counts every rank's units.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [0.25, 0.40][rank]   # seconds of device time on this rank

        def reduce_max(x):
            t = torch.tensor([x], dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            return float(t.item())

        value, t = bench.aggregate(local, 4096 * 10, world, reduce_max)
        seeds = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(seeds, torch.tensor([bench.rank_seed(2, rank)], dtype=torch.int64))
        out[rank] = (value, t, [int(s.item()) for s in seeds])
    finally:
        dist.destroy_process_group()


def test_weak_scaling_aggregation_two_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(2):
        value, t, seeds = res[r]
        assert t == pytest.approx(0.40)                      # the slowest rank sets the job time
        assert value == pytest.approx(2 * 4096 * 10 / 0.40)  # all ranks' queries count
        assert len(set(seeds)) == 2                          # independent requests per rank


def test_single_rank_aggregation():
    value, t = bench.aggregate(0.5, 100, 1)
    assert (value, t) == (200.0, 0.5)
