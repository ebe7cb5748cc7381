"""Key-list attention with sink and recent-window keys (lsa_sparse_attn_sw / _bwd) against the oracle.

A query attends to the union of its selected keys, the dense tail, the first n_sink positions
and the window of positions up to its own, each key once.  The windows below overlap the
selected leaves and the tail, so the de-duplication is exercised.  Tolerances as for the
other attention tests: fp32 max-abs 1e-4; bf16 max-abs 2e-2 and mean-abs 2e-3; gradients
relative to the reference's own scale.
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


def _tol(dtype):
    return (1e-4, 1e-4) if dtype == "f32" else (2e-2, 2e-3)


def _selected(lsa, cfg, case):
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "V", "W")}
    qp = case.q_pos.to(DEV)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx = lsa.select(tree, g["Q"], g["W"], cfg.beam, qp)
    return g, qp, idx


def _compare(lsa, cfg, case, g, qp, idx, tail, sink, window, heads=None):
    O, LSE = lsa.sparse_attn(g["Q"], g["K"], g["V"], idx, qp, True, tail, sink=sink, window=window)
    torch.cuda.synchronize()
    tmax, tmean = _tol(cfg.dtype)
    for h in (range(cfg.Hkv) if heads is None else heads):
        sl = slice(h * cfg.G, (h + 1) * cfg.G)
        hidx = None if idx is None else idx[h].cpu()
        Oo, Lo = orc.attn_fwd(case.Q[:, sl], case.K[h], case.V[h], hidx, q_pos=case.q_pos.numpy(), causal=True,
                              tail=tail, sink=sink, window=window)
        err = np.abs(O[:, sl].float().cpu().numpy() - Oo)
        assert err.max() <= tmax and err.mean() <= tmean, (h, sink, window, err.max(), err.mean())
        assert np.abs(LSE[:, sl].cpu().numpy() - Lo).max() <= 1e-3
    return O, LSE


def test_decode_shape_window_over_tail_and_tree(lsa):
    """decode_128k geometry: 24 steps whose windows cover the appended tail and reach back into
    positions that the selected leaves may also hold."""
    cfg = configs.get("decode_128k").scaled(Hkv=2, Hq=8, T=24)
    case = cfg.case("cpu")
    g, qp, idx = _selected(lsa, cfg, case)
    tail = (cfg.n, cfg.n_cap)
    for sink, window in ((4, 64), (0, 300), (16, 0), (1, 1)):
        _compare(lsa, cfg, case, g, qp, idx, tail, sink, window)


def test_prefill_shape_window_overlaps_leaves(lsa):
    """Causal chunk over a 4-level tree: each window (and the sink) overlaps selected leaves."""
    cfg = configs.get("prefill_1m").scaled(n=8 * 8 * 4 * 2 * 64, branching=(8, 8, 4, 2), beam=(4, 16, 16, 8),
                                           Hkv=2, Hq=8, T=256, comps=256)
    case = cfg.case("cpu")
    g, qp, idx = _selected(lsa, cfg, case)
    # how many selected keys also fall in the window: the de-duplication must matter here
    q = case.q_pos.numpy()[None, :, None]
    sel = idx.cpu().numpy()
    assert ((sel >= q - 127) & (sel <= q)).sum() > 0
    for sink, window in ((16, 128), (64, 512)):
        _compare(lsa, cfg, case, g, qp, idx, (0, 0), sink, window)


def test_fp32_and_no_index_list(lsa):
    """fp32 (d = 64), and a call without index lists: sink + window alone is local attention."""
    cfg = configs.get("tiny").scaled(T=64)
    case = cfg.case("cpu")
    n = cfg.n
    case.q_pos = torch.arange(n - 64, n, dtype=torch.int32)
    g, qp, idx = _selected(lsa, cfg, case)
    _compare(lsa, cfg, case, g, qp, idx, (0, 0), 4, 40)
    _compare(lsa, cfg, case, g, qp, None, (0, 0), 2, 100)


def test_backward_with_sink_and_window(lsa):
    """Training geometry, scaled (n = T = 8192, causal): dQ, dK, dV with sink and window keys."""
    cfg = configs.get("train_128k").scaled(n=8192, T=8192, branching=(8, 4, 4), beam=(4, 8, 8), Hkv=2, Hq=8,
                                           comps=64)
    case = cfg.case("cpu")
    g, qp, idx = _selected(lsa, cfg, case)
    sink, window = 4, 96
    O, LSE = _compare(lsa, cfg, case, g, qp, idx, (0, 0), sink, window)
    dO = case.dO.to(DEV)
    dQ, dK, dV = lsa.sparse_attn_bwd(g["Q"], g["K"], g["V"], O, LSE, dO, idx, qp, True, sink=sink, window=window)
    torch.cuda.synchronize()
    for h in range(cfg.Hkv):
        sl = slice(h * cfg.G, (h + 1) * cfg.G)
        oQ, oK, oV = orc.attn_bwd(case.Q[:, sl], case.K[h], case.V[h], idx[h].cpu(), case.dO[:, sl],
                                  q_pos=case.q_pos.numpy(), causal=True, sink=sink, window=window)
        for name, got, want in (("dQ", dQ[:, sl], oQ), ("dK", dK[h], oK), ("dV", dV[h], oV)):
            parity.check_grad(name, got.cpu().numpy(), want, zero_untouched=name != "dQ")


def test_rejects_bad_sink_window(lsa):
    Q = torch.zeros(2, 4, 128, dtype=torch.bfloat16, device=DEV)
    K = torch.zeros(1, 256, 128, dtype=torch.bfloat16, device=DEV)
    qp = torch.tensor([10, 20], dtype=torch.int32, device=DEV)
    with pytest.raises(lsa.LsaError) as e:
        lsa.sparse_attn(Q, K, K, None, qp, True, sink=-1, window=4)
    assert e.value.code == lsa.LSA_ERR_SHAPE
    with pytest.raises(lsa.LsaError) as e:
        lsa.sparse_attn(Q, K, K, None, qp, True, sink=300, window=4)   # sink beyond n_cap
    assert e.value.code == lsa.LSA_ERR_SHAPE


@pytest.mark.parametrize("G", [4, 1, 8])
def test_tree_attention_sink_window(lsa, G):
    """Leaf-by-leaf attention with sink and window keys (leaf keys inside them left out, the dense
    part merged as one more partial) = the key-list attention over the same union = the oracle."""
    cfg = configs.get("prefill_1m").scaled(n=8 * 8 * 4 * 2 * 64, branching=(8, 8, 4, 2), beam=(4, 16, 16, 8),
                                           Hkv=2, Hq=2 * G, T=300, comps=256)
    case = cfg.case("cpu", seed=21 + G)
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "V", "W")}
    qp = case.q_pos.to(DEV)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select(tree, g["Q"], g["W"], cfg.beam, qp, leaves=True)
    for sink, window in ((8, 96), (0, 64), (32, 0)):
        O, LSE = lsa.tree_attn(tree, g["Q"], g["K"], g["V"], leaves, qp, causal=True, sink=sink, window=window)
        O2, L2 = lsa.sparse_attn(g["Q"], g["K"], g["V"], idx, qp, True, sink=sink, window=window)
        torch.cuda.synchronize()
        d = (O.float() - O2.float()).abs()
        assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3, (G, sink, window, d.max().item())
        assert (LSE - L2).abs().max().item() <= 1e-3
        rows = np.arange(0, cfg.T, 37)
        h = 1
        sl = slice(h * G, (h + 1) * G)
        Oo, Lo = orc.attn_fwd(case.Q[rows][:, sl], case.K[h], case.V[h], idx[h][rows].cpu(),
                              q_pos=case.q_pos.numpy()[rows], causal=True, sink=sink, window=window)
        err = np.abs(O[rows][:, sl].float().cpu().numpy() - Oo)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3, (G, sink, window, err.max(), err.mean())
        assert np.abs(LSE[rows][:, sl].cpu().numpy() - Lo).max() <= 1e-3


def test_tree_attention_sink_window_fallback(lsa):
    """fp32, d = 64 (not the tensor-core path): expanded key lists with the sink and window."""
    cfg = configs.get("tiny").scaled(T=64)
    case = cfg.case("cpu")
    n = cfg.n
    case.q_pos = torch.arange(n - 64, n, dtype=torch.int32)
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "V", "W")}
    qp = case.q_pos.to(DEV)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select(tree, g["Q"], g["W"], cfg.beam, qp, leaves=True)
    O, LSE = lsa.tree_attn(tree, g["Q"], g["K"], g["V"], leaves, qp, causal=True, sink=3, window=50)
    torch.cuda.synchronize()
    Oo, Lo = orc.attn_fwd(case.Q, case.K[0], case.V[0], idx[0].cpu(), q_pos=case.q_pos.numpy(), causal=True,
                          sink=3, window=50)
    assert np.abs(O.cpu().numpy() - Oo).max() <= 1e-4
    assert np.abs(LSE.cpu().numpy() - Lo).max() <= 1e-4


def test_tree_attention_sink_window_scattered_queries(lsa):
    """Queries at scattered, unsorted positions (some inside the sink, some near position 0): the
    tiles' windows are disjoint, so the dense part must visit only the key blocks its rows need."""
    G = 4
    cfg = configs.get("prefill_1m").scaled(n=8 * 8 * 4 * 2 * 64, branching=(8, 8, 4, 2), beam=(4, 16, 16, 8),
                                           Hkv=2, Hq=2 * G, T=200, comps=256)
    case = cfg.case("cpu", seed=77)
    rng = np.random.default_rng(78)
    qpos = rng.choice(np.arange(cfg.n), size=cfg.T, replace=False)
    qpos[:4] = (0, 1, 5, 17)
    case.q_pos = torch.from_numpy(qpos.astype(np.int32))
    g = {k: getattr(case, k).to(DEV) for k in ("Q", "K", "V", "W")}
    qp = case.q_pos.to(DEV)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select(tree, g["Q"], g["W"], cfg.beam, qp, leaves=True)
    for sink, window in ((16, 200), (0, 1), (3, 0)):
        O, LSE = lsa.tree_attn(tree, g["Q"], g["K"], g["V"], leaves, qp, causal=True, sink=sink, window=window)
        O2, L2 = lsa.sparse_attn(g["Q"], g["K"], g["V"], idx, qp, True, sink=sink, window=window)
        torch.cuda.synchronize()
        d = (O.float() - O2.float()).abs()
        assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3, (sink, window, d.max().item())
        assert (LSE - L2).abs().max().item() <= 1e-3
        rows = np.concatenate([np.arange(4), np.arange(4, cfg.T, 29)])
        for h in range(cfg.Hkv):
            sl = slice(h * G, (h + 1) * G)
            Oo, Lo = orc.attn_fwd(case.Q[rows][:, sl], case.K[h], case.V[h], idx[h][rows].cpu(),
                                  q_pos=qpos[rows].astype(np.int32), causal=True, sink=sink, window=window)
            err = np.abs(O[rows][:, sl].float().cpu().numpy() - Oo)
            assert err.max() <= 2e-2 and err.mean() <= 2e-3, (h, sink, window, err.max(), err.mean())
            assert np.abs(LSE[rows][:, sl].cpu().numpy() - Lo).max() <= 1e-3
