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


def _head_split_worker(rank, world, port, out):
    """One request, KV heads split over the ranks: each rank builds the index of its own
    heads, selects and attends for its query heads (the CPU oracle stands in for the
    device), its tree descriptor comes from the C ABI's host-side call, and the outputs
    are gathered over gloo."""
    import numpy as np

    from hierarchical_latent_key_b200 import configs, lsa, shard
    from oracle import oracle as orc

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = configs.get("tiny").scaled(Hkv=3, Hq=6, T=40)
        case = cfg.case("cpu")
        Q, K, V, W = shard.local_inputs(case.Q, case.K, case.V, case.W, rank, world)
        lo, hi = shard.head_range(rank, world, cfg.Hkv)
        desc = lsa.lsa_tree_describe(hi - lo, cfg.r, cfg.branching, cfg.leaf)
        O = torch.zeros(cfg.T, Q.shape[1], cfg.d, dtype=torch.float64)
        for h in range(hi - lo):
            tree = orc.build_tree(orc.project(K[h, :cfg.n], W[h]), cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
            Qg = Q[:, h * cfg.G:(h + 1) * cfg.G]
            idx, _, _ = orc.select(orc.query_latent(Qg, W[h]), tree, cfg.beam)
            Oh, _ = orc.attn_fwd(Qg, K[h], V[h], idx)
            O[:, h * cfg.G:(h + 1) * cfg.G] = torch.from_numpy(np.asarray(Oh))
        full = shard.gather_heads(O, world, cfg.Hkv)
        out[rank] = (full.numpy(), int(desc.n_heads), int(desc.bytes), (lo, hi))
    finally:
        dist.destroy_process_group()


def test_kv_head_split_two_ranks():
    """3 KV heads over 2 ranks (2 + 1): the gathered output equals one process serving all
    heads, the per-rank index descriptors cover the ranks' heads, and the ranges tile."""
    import numpy as np

    from hierarchical_latent_key_b200 import configs, lsa, shard
    from oracle import oracle as orc

    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_head_split_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0
        res = dict(out)
    cfg = configs.get("tiny").scaled(Hkv=3, Hq=6, T=40)
    case = cfg.case("cpu")
    want = np.zeros((cfg.T, cfg.Hq, cfg.d))
    for h in range(cfg.Hkv):
        tree = orc.build_tree(orc.project(case.K[h, :cfg.n], case.W[h]), cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
        Qg = case.Q[:, h * cfg.G:(h + 1) * cfg.G]
        idx, _, _ = orc.select(orc.query_latent(Qg, case.W[h]), tree, cfg.beam)
        want[:, h * cfg.G:(h + 1) * cfg.G], _ = orc.attn_fwd(Qg, case.K[h], case.V[h], idx)
    whole = lsa.lsa_tree_describe(cfg.Hkv, cfg.r, cfg.branching, cfg.leaf)
    assert [res[r][3] for r in range(2)] == [(0, 2), (2, 3)]
    assert res[0][1] + res[1][1] == cfg.Hkv
    assert res[0][2] + res[1][2] >= whole.bytes >= max(res[0][2], res[1][2])
    for r in range(2):
        np.testing.assert_array_equal(res[r][0], want)   # same arithmetic, same order: bit-identical


def test_head_ranges_tile():
    from hierarchical_latent_key_b200 import shard
    for H in (1, 4, 7, 8):
        for world in (1, 2, 3, 8):
            if world > H:
                continue
            rs = [shard.head_range(r, world, H) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            assert max(hi - lo for lo, hi in rs) - min(hi - lo for lo, hi in rs) <= 1
