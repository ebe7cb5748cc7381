"""Index over pooled keys (lsa_build_tree_pooled) against the oracle.

Pooling (bdtechtalks.com, "Latent sparse attention", "How latent sparse attention works"): block
j of a head holds keys [j*p, (j+1)*p) and is represented by the mean of their latent rows; the
k-means levels cluster the blocks, and every leaf lists the keys of its blocks.  Checks:
  * every k-means round of the GPU build, recomputed by the oracle from the GPU's previous
    assignment over the oracle's pooled latents (float64): equal, or a stable assignment within
    the tolerance band;
  * the tree as a tree of keys: leaves are permutations of whole aligned blocks in ascending
    position, every centroid is the mean of the latent rows of the keys under its node (fp32
    relative 1e-5), min_pos is the smallest key position under the node;
  * without a differing round, the oracle's own pooled tree equals the GPU's exactly;
  * selection and leaf-by-leaf attention on the pooled index, stage-wise against the oracle.
"""
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


@pytest.mark.parametrize("pool,branching", [(4, (8, 8, 4, 2)), (2, (8, 8, 4, 2)), (64, (8, 4, 4))])
def test_pooled_build_select_attend(lsa, pool, branching):
    n = int(np.prod(branching)) * 64
    cfg = configs.get("prefill_1m").scaled(n=n, branching=branching, beam=(4, 16, 16, 8)[:len(branching)],
                                           Hkv=2, Hq=8, T=160, comps=256)
    case = cfg.case("cpu", seed=31 + pool)
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "V", "W")}
    qp = case.q_pos.to(DEV)
    tree, trace = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed, trace=True,
                                 pool=pool)
    idx, leaves, qlat, beams = lsa.select(tree, g["Q"], g["W"], cfg.beam, qp, qlat=True, beams=True, leaves=True)
    O, LSE = lsa.tree_attn(tree, g["Q"], g["K"], g["V"], leaves, qp, causal=True)
    torch.cuda.synchronize()
    qpn = case.q_pos.numpy()
    for h in range(cfg.Hkv):
        Z = orc.project(case.K[h, :n], case.W[h])
        Zp = orc.pool_keys(Z, pool)
        rd, _ = parity.check_build_stagewise(Zp, trace[:, :, h].cpu().numpy(), cfg.branching, cfg.leaf // pool,
                                             cfg.iters, cfg.seed)
        th = parity.export_tree(tree, h)
        parity.check_tree_structure(th, Z, cfg.leaf)
        blk = th["leaf_index"].astype(np.int64).reshape(-1, pool)
        assert np.all(blk[:, 0] % pool == 0) and np.all(blk == blk[:, :1] + np.arange(pool))
        if rd == 0:
            ot = orc.build_tree_pooled(Z, pool, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
            np.testing.assert_array_equal(th["leaf_index"], ot.leaf_index)
            for l in range(len(cfg.branching)):
                np.testing.assert_array_equal(th["min_pos"][l], ot.min_pos[l])
        oq = orc.query_latent(case.Q[:, h * cfg.G:(h + 1) * cfg.G], case.W[h])
        parity.check_select_stagewise(oq, th, cfg.branching, cfg.leaf, cfg.beam, qpn, beams[:, h].cpu().numpy(),
                                      idx[h].cpu().numpy())
        rows = np.arange(0, cfg.T, 7)
        Oo, Lo = orc.attn_fwd(case.Q[rows][:, h * cfg.G:(h + 1) * cfg.G], case.K[h], case.V[h],
                              idx[h][rows].cpu(), q_pos=qpn[rows], causal=True)
        err = np.abs(O[rows][:, h * cfg.G:(h + 1) * cfg.G].float().cpu().numpy() - Oo)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3, (pool, h, err.max(), err.mean())
        assert np.abs(LSE[rows][:, h * cfg.G:(h + 1) * cfg.G].cpu().numpy() - Lo).max() <= 1e-3


def test_pool_one_is_the_plain_build(lsa):
    cfg = configs.get("prefill_1m").scaled(n=8 * 8 * 4 * 64, branching=(8, 8, 4), beam=(4, 16, 8), Hkv=2, Hq=8,
                                           T=16, comps=128)
    case = cfg.case("cpu", seed=3)
    K, W = case.K.to(DEV), case.W.to(DEV)
    a = lsa.build_tree(K, W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    b = lsa.build_tree(K, W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed, pool=1)
    assert torch.equal(a.mem, b.mem)
