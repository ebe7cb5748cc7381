"""Flat search (lsa_select_flat) against the oracle: every eligible leaf scored, the n_leaves
best kept by (score desc, leaf id asc).  As for the beam walk, a kept set may differ from the
oracle's exact one only inside the near-tie band around the cut-off score (1e-5 relative)."""
import numpy as np
import pytest
import torch

from hierarchical_latent_key_b200 import configs
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def lsa():
    from hierarchical_latent_key_b200 import lsa as mod
    return mod


def _check_flat(qlat, tree_h, B, q_pos, got_leaves, got_idx, leaf, rows=None, rel=parity.NEAR_TIE_REL):
    """qlat [T, r] oracle latents; got_leaves [T, B]; got_idx [T, B * leaf]."""
    cents = np.asarray(tree_h["centroids"][-1], np.float64)
    mpos = np.asarray(tree_h["min_pos"][-1])
    li = np.asarray(tree_h["leaf_index"]).reshape(-1, leaf)
    near = 0
    for t in (range(qlat.shape[0]) if rows is None else rows):
        cand = np.arange(cents.shape[0])
        if q_pos is not None:
            cand = cand[mpos <= q_pos[t]]
        s = cents[cand] @ qlat[t]
        o = np.lexsort((cand, -s))
        k = min(B, len(cand))
        want = cand[o[:k]]
        row = np.asarray(got_leaves[t])
        got = row[row >= 0].astype(np.int64)
        assert len(got) == k and np.all(row[k:] == -1), (t, len(got), k)
        if set(got.tolist()) != set(want.tolist()):
            cutoff = s[o[k - 1]]
            floor = 1e-6 * np.linalg.norm(qlat[t]) * np.linalg.norm(cents[cand], axis=1).max()
            score = dict(zip(cand.tolist(), s.tolist()))
            for node in set(got.tolist()) ^ set(want.tolist()):
                assert abs(score[node] - cutoff) <= rel * abs(cutoff) + floor, (t, node)
            near += 1
        expect = np.full(got_idx.shape[1], -1, np.int64)
        expect[:len(got) * leaf] = li[got].reshape(-1)
        np.testing.assert_array_equal(np.asarray(got_idx[t]), expect)
    return near


def _run(lsa, cfg, B, seed=0, rows=None):
    case = cfg.case("cpu", seed=seed) if seed else cfg.case("cpu")
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "W")}
    qp = None if case.q_pos is None else case.q_pos.to(DEV)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves, qlat = lsa.select_flat(tree, g["Q"], g["W"], B, qp, qlat=True, leaves=True)
    torch.cuda.synchronize()
    near = 0
    for h in range(cfg.Hkv):
        th = parity.export_tree(tree, h)
        oq = orc.query_latent(case.Q[:, h * cfg.G:(h + 1) * cfg.G], case.W[h])
        np.testing.assert_allclose(qlat[:, h].cpu().numpy(), oq, rtol=1e-4, atol=1e-5)
        near += _check_flat(oq, th, B, None if case.q_pos is None else case.q_pos.numpy(), leaves[h].cpu().numpy(),
                            idx[h].cpu().numpy(), cfg.leaf, rows)
    return near


def test_flat_prefill_geometry_causal(lsa):
    """Causal chunk over 512 leaves: leaves whose smallest position lies past the query are
    not candidates."""
    cfg = configs.get("prefill_1m").scaled(n=8 * 8 * 4 * 2 * 64, branching=(8, 8, 4, 2), beam=(4, 16, 16, 8),
                                           Hkv=2, Hq=8, T=300, comps=256)
    for B in (8, 32, 1):
        print("near-ties", _run(lsa, cfg, B, seed=7))


def test_flat_decode_geometry(lsa):
    """2048 leaves per head (8 tiles), queries past the end of the index."""
    cfg = configs.get("decode_128k").scaled(Hkv=2, Hq=8, T=40)
    print("near-ties", _run(lsa, cfg, 32))


def test_flat_ragged_leaves(lsa):
    """960 leaves per head (the last 128-leaf tile of the tensor-core kernel is half full),
    two query heads per group, 200 causal queries (a partial query tile)."""
    cfg = configs.get("prefill_1m").scaled(n=8 * 8 * 5 * 3 * 64, branching=(8, 8, 5, 3), beam=(4, 16, 16, 7),
                                           Hkv=3, Hq=6, T=200, comps=128)
    for B in (7, 32):
        print("near-ties", _run(lsa, cfg, B, seed=11))


def test_flat_fp32_small(lsa):
    """fp32, d = 64, r = 16, 256 leaves, no positions; a partial last tile is not possible here,
    so a tree of 16 x 12 leaves (192) gives one."""
    cfg = configs.get("tiny")
    print("near-ties", _run(lsa, cfg, 8))
    cfg = configs.get("tiny").scaled(n=16 * 12 * 16, branching=(16, 12), beam=(4, 8))
    print("near-ties", _run(lsa, cfg, 8))


def test_flat_rejects_bad_budget(lsa):
    cfg = configs.get("tiny")
    case = cfg.case("cpu")
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "W")}
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, 2, 0)
    with pytest.raises(lsa.LsaError) as e:
        lsa.select_flat(tree, g["Q"], g["W"], 33)
    assert e.value.code == lsa.LSA_ERR_SHAPE
