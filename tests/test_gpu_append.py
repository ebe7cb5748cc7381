"""Update of the index on append (lsa_tree_append) against the oracle.

kongchang.com, "How LSA Sidesteps Per-Key Scoring with Hierarchical Clustering": the tree can be
precomputed and updated.  Once U = leaf * b_1 * ... * b_{L-1} keys are appended, they get a subtree
of their own (the plain build on those keys, positions counted from the block's first key),
attached as one more top-level node.  Checks after every append:
  * the subtree's k-means rounds, stage-wise against the oracle on the appended keys' latents;
  * old nodes unchanged (bitwise), new nodes after them on every level;
  * the grown tree as a tree of keys: centroids = means of the keys listed under each node (the
    new top node included), min_pos, ascending leaves, a permutation of all indexed positions;
  * without a differing round, the oracle's own append equals the GPU's;
  * selection and attention over the grown tree for decode queries in the appended block.
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


def _levels(tree, h):
    th = parity.export_tree(tree, h)
    return orc.Tree.from_levels(tree_branching(tree), tree.desc.leaf_size, th["centroids"], th["min_pos"],
                                th["leaf_index"]), th


def tree_branching(tree):
    return tuple(int(tree.desc.branching[l]) for l in range(tree.desc.levels))


def _append_and_check(lsa, cfg, case, g, tree):
    n = int(tree.desc.n_tree)
    grown, tr = lsa.tree_append(tree, g["K"], g["W"], cfg.iters, cfg.seed, trace=True)
    torch.cuda.synchronize()
    U = int(grown.desc.n_tree) - n
    br = tree_branching(tree)
    assert tree_branching(grown) == (br[0] + 1,) + br[1:]
    for l in range(tree.desc.levels):
        k = int(tree.desc.nodes[l])
        assert torch.equal(grown.centroids(l)[:, :k], tree.centroids(l))
        assert torch.equal(grown.min_pos(l)[:, :k], tree.min_pos(l))
    assert torch.equal(grown.leaf_index()[:, :n], tree.leaf_index())
    rounds = 0
    for h in range(cfg.Hkv):
        Znew = orc.project(case.K[h, n:n + U], case.W[h])
        rd, _ = parity.check_build_stagewise(Znew, tr[:, :, h].cpu().numpy(), br[1:], cfg.leaf, cfg.iters, cfg.seed)
        rounds += rd
        old, _ = _levels(tree, h)
        _, th = _levels(grown, h)
        parity.check_tree_structure(th, orc.project(case.K[h, :n + U], case.W[h]), cfg.leaf)
        if rd == 0:
            ot = orc.tree_append(old, Znew, cfg.iters, cfg.seed)
            np.testing.assert_array_equal(th["leaf_index"], ot.leaf_index)
            for l in range(len(br)):
                np.testing.assert_array_equal(th["min_pos"][l], ot.min_pos[l])
                scale = np.abs(ot.centroids[l]).max()
                assert np.abs(th["centroids"][l] - ot.centroids[l]).max() <= 1e-5 * scale
    return grown, rounds


def _select_and_attend(lsa, cfg, case, g, tree, rows):
    Q = g["Q"][rows]
    qp = torch.as_tensor(np.asarray(case.q_pos)[rows], dtype=torch.int32, device=DEV)
    idx, leaves, qlat, beams = lsa.select(tree, Q, g["W"], cfg.beam, qp, qlat=True, beams=True, leaves=True)
    O, LSE = lsa.sparse_attn(Q, g["K"], g["V"], idx, qp, True)
    torch.cuda.synchronize()
    qpn = qp.cpu().numpy()
    for h in range(cfg.Hkv):
        _, th = _levels(tree, h)
        oq = orc.query_latent(case.Q[rows][:, h * cfg.G:(h + 1) * cfg.G], case.W[h])
        parity.check_select_stagewise(oq, th, tree_branching(tree), cfg.leaf, cfg.beam, qpn,
                                      beams[:, h].cpu().numpy(), idx[h].cpu().numpy())
        Oo, Lo = orc.attn_fwd(case.Q[rows][:, h * cfg.G:(h + 1) * cfg.G], case.K[h], case.V[h], idx[h].cpu(),
                              q_pos=qpn, causal=True)
        err = np.abs(O[:, h * cfg.G:(h + 1) * cfg.G].float().cpu().numpy() - Oo)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3, (h, err.max(), err.mean())
        assert np.abs(LSE[:, h * cfg.G:(h + 1) * cfg.G].cpu().numpy() - Lo).max() <= 1e-3
    return idx


def test_append_two_subtrees_decode(lsa):
    """Tree 4/8/4, leaf 64 over 8192 keys; two appends of 2048 decode keys (top fan-out 4 -> 6),
    then decode queries in the second appended block select over the grown tree."""
    U = 8 * 4 * 64
    cfg = configs.get("decode_128k").scaled(n=4 * U, branching=(4, 8, 4), beam=(4, 16, 16), Hkv=2, Hq=8, T=2 * U,
                                            comps=128)
    case = cfg.case("cpu", seed=41)
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "V", "W")}
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    for _ in range(2):
        tree, _ = _append_and_check(lsa, cfg, case, g, tree)
    assert int(tree.desc.n_tree) == cfg.n + 2 * U
    _select_and_attend(lsa, cfg, case, g, tree, np.arange(2 * U - 48, 2 * U))


def test_append_top_level_past_32(lsa):
    """Tree 16/2, leaf 8 grown by 24 appends of 16 keys to 40 top nodes: level 0 then has more
    candidates than one warp holds (the select kernels' wider sort); both select kernels
    (small batch and warp per query) agree with each other and with the oracle."""
    U = 2 * 8
    cfg = configs.get("decode_128k").scaled(n=16 * U, branching=(16, 2), leaf=8, beam=(12, 8), Hkv=2, Hq=8,
                                            T=24 * U, comps=32)
    case = cfg.case("cpu", seed=43)
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "V", "W")}
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    diff = 0
    for _ in range(24):
        tree, rd = _append_and_check(lsa, cfg, case, g, tree)
        diff += rd
    assert int(tree.desc.nodes[0]) == 40
    rows = np.arange(cfg.T - 40, cfg.T)
    idx_small = _select_and_attend(lsa, cfg, case, g, tree, rows)
    # the same queries inside a batch large enough for the warp-per-query kernel
    big = np.concatenate([np.arange(cfg.T)] * 3)
    qp = torch.as_tensor(np.asarray(case.q_pos)[big], dtype=torch.int32, device=DEV)
    idx_big = lsa.select(tree, g["Q"][big], g["W"], cfg.beam, qp)
    torch.cuda.synchronize()
    assert torch.equal(idx_big[:, cfg.T - 40:cfg.T], idx_small)


def test_decode_loop_with_updates(lsa):
    """Decode over a 4/8/4 index: each step's key joins the dense tail before the step attends;
    when the tail holds U keys they are attached as a subtree (lsa_tree_append) and the tail
    restarts after them.  Sampled steps around both updates: selection stage-wise against the
    oracle on the grown index, attention over (selected keys + tail) against the oracle."""
    U = 8 * 4 * 64
    cfg = configs.get("decode_128k").scaled(n=4 * U, branching=(4, 8, 4), beam=(4, 16, 16), Hkv=2, Hq=8,
                                            T=2 * U + 40, comps=128)
    case = cfg.case("cpu", seed=47)
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "V", "W")}
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    tail_begin = cfg.n
    sample = {0, 1, U - 2, U - 1, U, U + 1, 2 * U - 1, 2 * U, 2 * U + 39}
    updates = 0
    for s in range(cfg.T):
        p = cfg.n + s                          # the step's key, appended before it attends
        if p - tail_begin + 1 == U:            # the tail holds a full block: grow the index
            assert int(tree.desc.n_tree) == tail_begin
            tree = lsa.tree_append(tree, g["K"], g["W"], cfg.iters, cfg.seed)
            tail_begin = p + 1
            updates += 1
        if s not in sample:
            continue
        qp = torch.tensor([p], dtype=torch.int32, device=DEV)
        idx, qlat, beams = lsa.select(tree, g["Q"][s:s + 1], g["W"], cfg.beam, qp, qlat=True, beams=True)
        tail = (tail_begin, p + 1)
        O, LSE = lsa.sparse_attn(g["Q"][s:s + 1], g["K"], g["V"], idx, qp, True, tail)
        torch.cuda.synchronize()
        for h in range(cfg.Hkv):
            _, th = _levels(tree, h)
            Qg = case.Q[s:s + 1, h * cfg.G:(h + 1) * cfg.G]
            oq = orc.query_latent(Qg, case.W[h])
            parity.check_select_stagewise(oq, th, tree_branching(tree), cfg.leaf, cfg.beam, np.array([p]),
                                          beams[:, h].cpu().numpy(), idx[h].cpu().numpy())
            Oo, Lo = orc.attn_fwd(Qg, case.K[h], case.V[h], idx[h].cpu(), q_pos=np.array([p], np.int32),
                                  causal=True, tail=tail)
            err = np.abs(O[:, h * cfg.G:(h + 1) * cfg.G].float().cpu().numpy() - Oo)
            assert err.max() <= 2e-2 and err.mean() <= 2e-3, (s, h, err.max(), err.mean())
            assert np.abs(LSE[:, h * cfg.G:(h + 1) * cfg.G].cpu().numpy() - Lo).max() <= 1e-3
    assert updates == 2 and int(tree.desc.nodes[0]) == 6
