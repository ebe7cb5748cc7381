"""Full-size workloads on the GPU, checked against the oracle on sampled outputs.

Each test runs the CUDA path in the launch configuration bench.py times (tree build,
select, tree or key-list attention; decode with the dense tail) at the workload's full
size, then checks (a) properties that hold at any size (balanced leaves, permutation,
centroid = mean of members on sampled nodes) and (b) sampled outputs the oracle computes
one by one: k-means rounds of sampled parent nodes (stage-wise), the beam walk of sampled
queries (stage-wise, near-tie band), and attention of sampled queries on the GPU's keys.
"""
import math

import numpy as np
import pytest
import torch

from hierarchical_latent_key_b200 import configs
from oracle import oracle as orc
from tests import parity

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"


@pytest.fixture(scope="module")
def lsa():
    from hierarchical_latent_key_b200 import lsa as mod
    return mod


def _rows(K, h, ids):
    """Float64 copies of rows `ids` of head h of a (device) key/value tensor."""
    t = torch.as_tensor(np.asarray(ids), dtype=torch.int64, device=K.device)
    return K[h].index_select(0, t).double().cpu().numpy()


def _tree_props(tree, h, K, W_h, n, leaf, rng, n_nodes=24):
    """Permutation, ascending leaves, and centroid = mean of members for sampled nodes."""
    li = tree.leaf_index()[h].cpu().numpy().astype(np.int64)
    assert np.array_equal(np.sort(li), np.arange(n))
    assert np.all(np.diff(li.reshape(-1, leaf), axis=1) > 0)
    for l in range(tree.levels):
        nodes = tree.desc.nodes[l]
        per = n // nodes
        pick = rng.choice(nodes, min(n_nodes, nodes), replace=False)
        cent = tree.centroids(l)[h].cpu().numpy()
        mpos = tree.min_pos(l)[h].cpu().numpy()
        for node in pick:
            members = li[node * per:(node + 1) * per]
            Z = orc.project(_rows(K, h, members), W_h)
            mu = Z.mean(axis=0)
            assert np.abs(cent[node] - mu).max() <= 1e-5 * np.abs(mu).max() + 1e-6, (l, node)
            assert mpos[node] == members.min()


def _check_queries(case, cfg, tree, h, rows, q_pos, beams, idx, O, LSE, tail=(0, 0)):
    """Stage-wise select and attention for query rows `rows` of head h (CPU case)."""
    th = parity.export_tree(tree, h)
    Qg = case.Q[rows][:, h * cfg.G:(h + 1) * cfg.G]
    oq = orc.query_latent(Qg, case.W[h].cpu())
    qp = None if q_pos is None else q_pos[rows]
    near = parity.check_select_stagewise(oq, th, cfg.branching, cfg.leaf, cfg.beam, qp,
                                         beams[:, h][:, rows].cpu().numpy(), idx[h][rows].cpu().numpy())
    Oo, Lo = orc.attn_fwd(Qg, case.K[h].cpu(), case.V[h].cpu(), idx[h][rows].cpu(), q_pos=qp,
                          causal=q_pos is not None, tail=tail)
    mx, mean = parity.attn_errors(O[rows][:, h * cfg.G:(h + 1) * cfg.G].float().cpu(), Oo)
    assert mx <= 2e-2 and mean <= 2e-3, (h, mx, mean)
    assert np.abs(LSE[rows][:, h * cfg.G:(h + 1) * cfg.G].cpu().numpy() - Lo).max() <= 1e-3
    return near


def test_decode_128k_all_heads(lsa):
    """All 8 KV heads, n = 131072, 256 decode steps (batched: causal by position, tail of
    appended keys).  Build checked stage-wise on two heads (sampled deep nodes)."""
    cfg = configs.get("decode_128k")
    case = cfg.case("cpu")
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "V", "W", "q_pos")}
    tree, trace = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed, trace=True)
    idx, beams = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], beams=True)
    O, LSE = lsa.sparse_attn(g["Q"], g["K"], g["V"], idx, g["q_pos"], True, (cfg.n, cfg.n_cap))
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    qp = case.q_pos.numpy()
    for h in (0, 5):
        Z = orc.project(case.K[h, :cfg.n], case.W[h])
        parity.check_build_stagewise(Z, trace[:, :, h].cpu().numpy(), cfg.branching, cfg.leaf, cfg.iters,
                                     cfg.seed, max_segments=8, rng=rng,
                                     check=lambda l, t, m: l > 0 or t in (0, cfg.iters - 1))
    near = 0
    for h in range(cfg.Hkv):
        _tree_props(tree, h, case.K, case.W[h].float().numpy(), cfg.n, cfg.leaf, rng, n_nodes=6)
        near += _check_queries(case, cfg, tree, h, np.arange(cfg.T), qp, beams, idx, O, LSE,
                               tail=(cfg.n, cfg.n_cap))
    print("decode_128k near-ties", near)


def test_prefill_1m_full(lsa):
    """1,048,576 cached keys, 4096-query causal chunk through select + tree attention."""
    cfg = configs.get("prefill_1m")
    case = cfg.case(DEV)
    tree, trace = lsa.build_tree(case.K, case.W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed, trace=True)
    idx, leaves, beams = lsa.select(tree, case.Q, case.W, cfg.beam, case.q_pos, beams=True, leaves=True)
    # the batched schedule (the one bench.py times) returns the same lists bit for bit
    idx_b, leaves_b, beams_b = lsa.select(tree, case.Q, case.W, cfg.beam, case.q_pos, beams=True, leaves=True,
                                          batched=True)
    O, LSE = lsa.tree_attn(tree, case.Q, case.K, case.V, leaves, case.q_pos, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(idx_b, idx) and torch.equal(leaves_b, leaves) and torch.equal(beams_b, beams)
    del idx_b, leaves_b, beams_b
    rng = np.random.default_rng(1)
    qp = case.q_pos.cpu().numpy()
    rows = np.sort(rng.choice(cfg.T, 48, replace=False))
    near = 0
    for h in (0, 3, 7):
        Kh = case.K[h].double().cpu().numpy()
        Vh = case.V[h].double().cpu().numpy()
        Wh = case.W[h].double().cpu().numpy()
        if h == 3:
            Z = orc.project(Kh[:cfg.n], Wh)
            parity.check_build_stagewise(Z, trace[:, :, h].cpu().numpy(), cfg.branching, cfg.leaf, cfg.iters,
                                         cfg.seed, max_segments=4, rng=rng,
                                         check=lambda l, t, m: m <= 65536 and t in (0, 4, 9))
            del Z
        _tree_props(tree, h, case.K, Wh, cfg.n, cfg.leaf, rng, n_nodes=8)
        th = parity.export_tree(tree, h)
        Qg = case.Q[rows][:, h * cfg.G:(h + 1) * cfg.G].double().cpu().numpy()
        oq = orc.query_latent(Qg, Wh)
        near += parity.check_select_stagewise(oq, th, cfg.branching, cfg.leaf, cfg.beam, qp[rows],
                                              beams[:, h][:, rows].cpu().numpy(), idx[h][rows].cpu().numpy())
        Oo, Lo = orc.attn_fwd(Qg, Kh, Vh, idx[h][rows].cpu(), q_pos=qp[rows], causal=True)
        mx, mean = parity.attn_errors(O[rows][:, h * cfg.G:(h + 1) * cfg.G].float().cpu(), Oo)
        assert mx <= 2e-2 and mean <= 2e-3, (h, mx, mean)
        assert np.abs(LSE[rows][:, h * cfg.G:(h + 1) * cfg.G].cpu().numpy() - Lo).max() <= 1e-3
        del Kh, Vh
    print("prefill_1m near-ties", near)


def test_decode_10m_full(lsa):
    """10,485,760 indexed keys, all 128 decode steps (lsa_decode_step: append, select, attention
    over the kept leaves and the dense tail, one step at a time as bench.py runs them), every step checked on all 8
    KV heads: the beam walk stage-wise (near-tie band), the key list exactly, attention on
    the GPU's keys.  The build is checked stage-wise on sampled segments of one head (every
    round of the three lowest levels) and by tree properties on every head."""
    cfg = configs.get("decode_10m")
    case = cfg.case(DEV)
    n = cfg.n
    Knew = case.K[:, n:].transpose(0, 1).clone(memory_format=torch.contiguous_format)       # rows the steps append
    Vnew = case.V[:, n:].transpose(0, 1).clone(memory_format=torch.contiguous_format)
    case.K[:, n:].zero_()
    case.V[:, n:].zero_()
    tree, trace = lsa.build_tree(case.K, case.W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed, trace=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(2)
    hb = 6
    W_b = case.W[hb].double().cpu().numpy()
    tr = trace[:, :, hb].cpu().numpy()
    del trace
    rd, kd = parity.check_build_stagewise(lambda pos: orc.project(_rows(case.K, hb, pos), W_b), tr, cfg.branching,
                                          cfg.leaf, cfg.iters, cfg.seed, max_segments=4, rng=rng,
                                          check=lambda l, t, m: m <= 81920)
    del tr
    print("decode_10m build rounds differing", rd, "keys", kd)
    for h in range(cfg.Hkv):
        _tree_props(tree, h, case.K, case.W[h].double().cpu().numpy(), n, cfg.leaf, rng, n_nodes=4)
    # the decode loop on the GPU as bench.py runs it: one lsa_decode_step per token (append,
    # select, attention); the select call alone gives the per-level beams for the stage-wise check
    dec = lsa.DecodeStep(tree, case.W, cfg.beam, case.K, cfg.Hq, cfg.T)
    st_idx, st_beams, st_O, st_LSE = [], [], [], []
    for s in range(cfg.T):
        Qs = case.Q[s:s + 1]
        O, LSE = dec.step(case.K, case.V, Qs, Knew[s], Vnew[s], n + s, n)
        idx, leaves, beams = lsa.select(tree, Qs, case.W, cfg.beam, case.q_pos[s:s + 1], beams=True, leaves=True)
        assert torch.equal(dec.leaves, leaves[:, 0]), s
        st_idx.append(idx.cpu()); st_beams.append(beams.cpu()); st_O.append(O.float().cpu()); st_LSE.append(LSE.cpu())
    assert lsa.lsa_status_check(dec.status) == lsa.LSA_OK
    torch.cuda.synchronize()
    near = 0
    for h in range(cfg.Hkv):
        th = parity.export_tree(tree, h)
        W_h = case.W[h].double().cpu().numpy()
        sl = slice(h * cfg.G, (h + 1) * cfg.G)
        for s in range(cfg.T):
            p = n + s
            Qg = case.Q[s:s + 1, sl].double().cpu().numpy()
            oq = orc.query_latent(Qg, W_h)
            near += parity.check_select_stagewise(oq, th, cfg.branching, cfg.leaf, cfg.beam, np.array([p]),
                                                  st_beams[s][:, h].numpy(), st_idx[s][h].numpy())
            # every selected key and every tail key precedes the query: compact them (non-causal)
            sel = st_idx[s][h, 0].numpy()
            keys = np.concatenate([sel[sel >= 0], np.arange(n, p + 1)])
            Kc, Vc = _rows(case.K, h, keys), _rows(case.V, h, keys)
            n_sel = int((sel >= 0).sum())
            Oo, Lo = orc.attn_fwd(Qg, Kc, Vc, np.arange(n_sel, dtype=np.int32)[None], tail=(n_sel, len(keys)))
            mx, mean = parity.attn_errors(st_O[s][:, sl], Oo)
            assert mx <= 2e-2 and mean <= 2e-3, (h, s, mx, mean)
            assert np.abs(st_LSE[s][:, sl].numpy() - Lo).max() <= 1e-3
    print("decode_10m near-ties", near, "of", cfg.T * cfg.Hkv * len(cfg.branching), "(query, head, level) beams")
    assert near <= cfg.T * cfg.Hkv * len(cfg.branching) // 100


def test_train_128k_full(lsa):
    """131072-token causal layer: build, select, tree-attention forward and backward; oracle on
    sampled queries (dQ, O) and sampled keys (dK, dV from every query that selected them)."""
    cfg = configs.get("train_128k")
    case = cfg.case(DEV)
    tree = lsa.build_tree(case.K, case.W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select(tree, case.Q, case.W, cfg.beam, case.q_pos, leaves=True)
    O, LSE = lsa.tree_attn(tree, case.Q, case.K, case.V, leaves, case.q_pos, causal=True)
    dQ, dK, dV = lsa.tree_attn_bwd(tree, case.Q, case.K, case.V, O, LSE, case.dO, leaves, case.q_pos, causal=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    h = 1
    sl = slice(h * cfg.G, (h + 1) * cfg.G)
    Qh = case.Q[:, sl].float().cpu().numpy()
    Kh = case.K[h].float().cpu().numpy()
    Vh = case.V[h].float().cpu().numpy()
    dOh = case.dO[:, sl].float().cpu().numpy()
    qp = case.q_pos.cpu().numpy()
    ih = idx[h].cpu().numpy()
    rows = np.sort(rng.choice(cfg.T, 64, replace=False))
    Oo, Lo = orc.attn_fwd(Qh[rows], Kh, Vh, ih[rows], q_pos=qp[rows], causal=True)
    mx, mean = parity.attn_errors(O[rows][:, sl].float().cpu(), Oo)
    assert mx <= 2e-2 and mean <= 2e-3, (mx, mean)
    oQ, _, _ = orc.attn_bwd(Qh[rows], Kh, Vh, ih[rows], dOh[rows], q_pos=qp[rows], causal=True)
    parity.check_grad("dQ", dQ[rows][:, sl].cpu().numpy(), oQ, zero_untouched=False)
    # dK, dV of every key of 8 sampled leaves (512 keys): a leaf is selected whole, so the
    # queries that listed its first key are every query that sees any of its keys
    li = tree.leaf_index()[h].cpu().numpy().reshape(-1, cfg.leaf)
    got_K, got_V, want_K, want_V = [], [], [], []
    for leaf in rng.choice(li.shape[0], 8, replace=False):
        keys = li[leaf]
        users = np.nonzero((ih == keys[0]).any(axis=1))[0]
        if len(users) == 0:
            continue
        _, oK, oV = orc.attn_bwd(Qh[users], Kh, Vh, ih[users], dOh[users], q_pos=qp[users], causal=True)
        got_K.append(dK[h, keys].cpu().numpy()); want_K.append(oK[keys])
        got_V.append(dV[h, keys].cpu().numpy()); want_V.append(oV[keys])
    assert len(got_K) >= 4
    parity.check_grad("dK", np.concatenate(got_K), np.concatenate(want_K))
    parity.check_grad("dV", np.concatenate(got_V), np.concatenate(want_V))


def test_tree_attention_beyond_partial_budget(lsa):
    """Above 24 GiB of per-(row, leaf) partials the tree attention takes its two-pass schedule
    (statistics, then outputs with fp32 red-adds): 131072 causal queries x 32 heads x 32 leaves
    (34 GB of partials).  Checked against the key-list attention on every row and against the
    oracle on sampled rows."""
    cfg = configs.get("train_128k").scaled(Hq=32)
    assert cfg.T * cfg.Hq * cfg.beam[-1] * 128 * 2 > (24 << 30)
    case = cfg.case(DEV)
    tree = lsa.build_tree(case.K, case.W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select(tree, case.Q, case.W, cfg.beam, case.q_pos, leaves=True)
    O, LSE = lsa.tree_attn(tree, case.Q, case.K, case.V, leaves, case.q_pos, causal=True)
    O2, L2 = lsa.sparse_attn(case.Q, case.K, case.V, idx, case.q_pos, True)
    torch.cuda.synchronize()
    d = (O.float() - O2.float()).abs()
    assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3
    assert (LSE - L2).abs().max().item() <= 1e-3
    rng = np.random.default_rng(5)
    h = 2
    sl = slice(h * cfg.G, (h + 1) * cfg.G)
    rows = np.sort(rng.choice(cfg.T, 32, replace=False))
    Oo, Lo = orc.attn_fwd(case.Q[rows][:, sl].double().cpu().numpy(), case.K[h].double().cpu().numpy(),
                          case.V[h].double().cpu().numpy(), idx[h][rows].cpu().numpy(),
                          q_pos=case.q_pos.cpu().numpy()[rows], causal=True)
    mx, mean = parity.attn_errors(O[rows][:, sl].float().cpu(), Oo)
    assert mx <= 2e-2 and mean <= 2e-3, (mx, mean)


def test_flat_prefill_1m_sampled(lsa):
    """Flat search over the 16384 leaves of each head at 1,048,576 keys, 4096 causal queries;
    the oracle checks sampled queries of two heads."""
    from tests.test_gpu_flat import _check_flat
    cfg = configs.get("prefill_1m")
    case = cfg.case(DEV)
    tree = lsa.build_tree(case.K, case.W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select_flat(tree, case.Q, case.W, cfg.beam[-1], case.q_pos, leaves=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    rows = np.sort(rng.choice(cfg.T, 48, replace=False))
    qp = case.q_pos.cpu().numpy()
    for h in (0, 5):
        th = parity.export_tree(tree, h)
        oq = orc.query_latent(case.Q[:, h * cfg.G:(h + 1) * cfg.G].double().cpu().numpy(), case.W[h].double().cpu().numpy())
        _check_flat(oq, th, cfg.beam[-1], qp, leaves[h].cpu().numpy(), idx[h].cpu().numpy(), cfg.leaf, rows)
