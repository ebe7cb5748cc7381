"""CUDA path vs the CPU oracle on the same seeded inputs (all through the C ABI).

Tolerances: selection bit-exact except near-ties within 1e-5 relative of the
cut-off score (counted); attention max-abs 1e-4 for fp32 inputs, max-abs 2e-2
and mean-abs 2e-3 for bf16 inputs (bf16 output rounding is ~4e-3 at |O| ~ 1).
"""
import math

import numpy as np
import pytest
import torch

from hierarchical_latent_key_b200 import configs, synth
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def lsa():
    from hierarchical_latent_key_b200 import lsa as mod
    return mod


def _check_grad(name, got, want):
    parity.check_grad(name, got, want, zero_untouched=name != "dQ")


def _tol(dtype):
    return (1e-4, 1e-4) if dtype == "f32" else (2e-2, 2e-3)


def _to(case, dev=DEV):
    return {k: (getattr(case, k).to(dev) if getattr(case, k) is not None else None)
            for k in ("Q", "K", "V", "W", "q_pos", "dO")}


def _run_case(lsa, cfg, case, heads_checked=None, max_segments=None, steps_tail=False):
    """Build, select and attend on the GPU; check each stage against the oracle."""
    g = _to(case)
    tree, trace = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed, trace=True)
    idx, qlat, beams = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], qlat=True, beams=True)
    tail = (cfg.n, cfg.n_cap) if steps_tail else (0, 0)
    O, LSE = lsa.sparse_attn(g["Q"], g["K"], g["V"], idx, g["q_pos"], cfg.causal, tail)
    torch.cuda.synchronize()
    report = dict(build_rounds_diff=0, build_keys_diff=0, near_ties=0)
    heads = range(cfg.Hkv) if heads_checked is None else heads_checked
    qp = None if case.q_pos is None else case.q_pos.numpy()
    for h in heads:
        Z = orc.project(case.K[h, :cfg.n], case.W[h])
        rd, kd = parity.check_build_stagewise(Z, trace[:, :, h].cpu().numpy(), cfg.branching, cfg.leaf,
                                              cfg.iters, cfg.seed, max_segments=max_segments)
        report["build_rounds_diff"] += rd
        report["build_keys_diff"] += kd
        th = parity.export_tree(tree, h)
        parity.check_tree_structure(th, Z, cfg.leaf)
        Qg = case.Q[:, h * cfg.G:(h + 1) * cfg.G]
        oq = orc.query_latent(Qg, case.W[h])
        np.testing.assert_allclose(qlat[:, h].cpu().numpy(), oq, rtol=1e-4, atol=1e-5)
        report["near_ties"] += parity.check_select_stagewise(
            oq, th, cfg.branching, cfg.leaf, cfg.beam, qp, beams[:, h].cpu().numpy(), idx[h].cpu().numpy())
        Oo, Lo = orc.attn_fwd(Qg, case.K[h], case.V[h], idx[h].cpu(), q_pos=qp, causal=cfg.causal, tail=tail)
        mx, mean = parity.attn_errors(O[:, h * cfg.G:(h + 1) * cfg.G].float().cpu(), Oo)
        tmax, tmean = _tol(cfg.dtype)
        assert mx <= tmax and mean <= tmean, (h, mx, mean)
        lse_err = np.abs(LSE[:, h * cfg.G:(h + 1) * cfg.G].cpu().numpy() - Lo).max()
        assert lse_err <= 1e-3, lse_err
    return tree, idx, O, LSE, report


def test_tiny_end_to_end(lsa):
    """The tiny fp32 workload end to end: the oracle builds its own tree and selects from
    scratch; the GPU must agree exactly (every k-means round, the tree, every selected key,
    no near-tie) and the attention over the oracle's own selection within 1e-4."""
    cfg = configs.get("tiny")
    case = cfg.case("cpu")
    tree, idx, O, LSE, rep = _run_case(lsa, cfg, case)
    Z = orc.project(case.K[0], case.W[0])
    otree = orc.build_tree(Z, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    oq = orc.query_latent(case.Q[:, 0:1], case.W[0])
    oidx, _, _ = orc.select(oq, otree, cfg.beam)
    print("tiny report", rep)
    assert rep["build_rounds_diff"] == 0 and rep["build_keys_diff"] == 0, rep
    assert rep["near_ties"] == 0, rep
    np.testing.assert_array_equal(tree.leaf_index()[0].cpu().numpy(), otree.leaf_index)
    for l in range(len(cfg.branching)):
        np.testing.assert_array_equal(tree.min_pos(l)[0].cpu().numpy(), otree.min_pos[l])
        np.testing.assert_allclose(tree.centroids(l)[0].cpu().numpy(), otree.centroids[l], rtol=1e-5, atol=1e-6)
    np.testing.assert_array_equal(idx[0].cpu().numpy(), oidx)
    Oo, Lo = orc.attn_fwd(case.Q, case.K[0], case.V[0], oidx)
    assert np.abs(O.cpu().numpy() - Oo).max() <= 1e-4
    assert np.abs(LSE.cpu().numpy() - Lo).max() <= 1e-4


def test_decode_shape_two_heads(lsa):
    """decode_128k geometry (n = 131072, tree 16/16/8, leaf 64) on 2 KV heads; 24 decode
    steps run as one causal batch whose tail holds the appended keys."""
    cfg = configs.get("decode_128k").scaled(Hkv=2, Hq=8, T=24)
    case = cfg.case("cpu")
    *_, rep = _run_case(lsa, cfg, case, max_segments=24, steps_tail=True)
    print("decode report", rep)


def test_prefill_shape_small(lsa):
    """Last-chunk prefill geometry, scaled: 4-level tree over 32768 keys, causal chunk of 384."""
    cfg = configs.get("prefill_1m").scaled(n=8 * 8 * 4 * 2 * 64, branching=(8, 8, 4, 2), beam=(4, 16, 16, 8),
                                           Hkv=2, Hq=8, T=384, comps=256)
    case = cfg.case("cpu")
    *_, rep = _run_case(lsa, cfg, case, max_segments=32)
    print("prefill report", rep)


def test_train_shape_small_fwd_bwd(lsa):
    """Training geometry, scaled: causal over n = T = 8192, tree (8, 4, 4), forward + backward."""
    cfg = configs.get("train_128k").scaled(n=8192, T=8192, branching=(8, 4, 4), beam=(4, 8, 8), Hkv=2, Hq=8,
                                           comps=64)
    case = cfg.case("cpu")
    tree, idx, O, LSE, rep = _run_case(lsa, cfg, case, max_segments=16)
    g = _to(case)
    dQ, dK, dV = lsa.sparse_attn_bwd(g["Q"], g["K"], g["V"], O, LSE, g["dO"], idx, g["q_pos"], True)
    torch.cuda.synchronize()
    qp = case.q_pos.numpy()
    for h in range(cfg.Hkv):
        sl = slice(h * cfg.G, (h + 1) * cfg.G)
        # the oracle uses the GPU's bf16 forward output only through the selection
        oQ, oK, oV = orc.attn_bwd(case.Q[:, sl], case.K[h], case.V[h], idx[h].cpu(), case.dO[:, sl],
                                  q_pos=qp, causal=True)
        for name, got, want in (("dQ", dQ[:, sl], oQ), ("dK", dK[h], oK), ("dV", dV[h], oV)):
            _check_grad(name, got.cpu().numpy(), want)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d,G", [(64, 1), (128, 4), (64, 8), (128, 2)])
@pytest.mark.parametrize("T", [1, 3, 700])
def test_attention_shapes_and_edges(lsa, dtype, d, G, T):
    """Split (few queries) and unsplit paths, ragged key counts, -1 pads, tail, causal."""
    torch.manual_seed(T * 100 + d + G)
    Hkv, n_cap, K_sel = 2, 3000, 203
    dt = synth.torch_dtype(dtype)
    Q = torch.randn(T, Hkv * G, d).to(dt)
    K = torch.randn(Hkv, n_cap, d).to(dt)
    V = torch.randn(Hkv, n_cap, d).to(dt)
    idx = torch.stack([torch.stack([torch.randperm(2500)[:K_sel] for _ in range(T)]) for _ in range(Hkv)]).int()
    idx[:, :, -7:] = -1
    q_pos = torch.randint(1200, n_cap, (T,), dtype=torch.int32)
    tail = (2600, 2777)
    for causal in (False, True):
        O, LSE = lsa.sparse_attn(Q.cuda(), K.cuda(), V.cuda(), idx.cuda(), q_pos.cuda(), causal, tail)
        for h in range(Hkv):
            sl = slice(h * G, (h + 1) * G)
            Oo, Lo = orc.attn_fwd(Q[:, sl], K[h], V[h], idx[h], q_pos=q_pos.numpy(), causal=causal, tail=tail)
            mx, mean = parity.attn_errors(O[:, sl].float().cpu(), Oo)
            tmax, tmean = _tol(dtype)
            assert mx <= tmax and mean <= tmean, (causal, h, mx, mean)
            assert np.abs(LSE[:, sl].cpu().numpy() - Lo).max() <= 1e-3


def test_attention_empty_and_all_masked(lsa):
    Q = torch.randn(0, 4, 128, dtype=torch.bfloat16, device=DEV)
    K = torch.randn(1, 64, 128, dtype=torch.bfloat16, device=DEV)
    O, LSE = lsa.sparse_attn(Q, K, K, torch.zeros(1, 0, 8, dtype=torch.int32, device=DEV))
    assert O.shape == (0, 4, 128)
    Q = torch.randn(3, 4, 128, dtype=torch.bfloat16, device=DEV)
    idx = torch.full((1, 3, 8), -1, dtype=torch.int32, device=DEV)
    O, LSE = lsa.sparse_attn(Q, K, K, idx)
    assert torch.all(O == 0) and torch.all(torch.isneginf(LSE))


def test_select_full_beam_is_flat_search(lsa):
    """With every node kept above the leaf level, the walk equals flat top-B over all leaves."""
    cfg = configs.get("tiny")
    case = cfg.case("cpu")
    g = _to(case)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    beam = (cfg.nodes[0], 8)
    idx, qlat = lsa.select(tree, g["Q"], g["W"], beam, None, qlat=True)
    leafc = tree.centroids(1)[0].double().cpu().numpy()
    s = qlat[:, 0].double().cpu().numpy() @ leafc.T
    li = tree.leaf_index()[0].cpu().numpy().reshape(-1, cfg.leaf)
    near = 0
    for t in range(cfg.T):
        o = np.lexsort((np.arange(s.shape[1]), -s[t]))[:8]
        want = li[o].reshape(-1)
        got = idx[0, t].cpu().numpy()
        if not np.array_equal(got, want):
            near += 1
            cutoff = s[t, o[-1]]
            got_leaves = {int(np.nonzero((li == k).any(1))[0][0]) for k in got[::cfg.leaf]}
            for node in got_leaves ^ set(o.tolist()):
                assert abs(s[t, node] - cutoff) <= 1e-5 * abs(cutoff) + 1e-6
    assert near <= 2


def test_build_deterministic(lsa):
    cfg = configs.get("decode_128k").scaled(Hkv=1, Hq=4)
    case = cfg.case("cpu")
    g = _to(case)
    t1 = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, 3, 7)
    t2 = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, 3, 7)
    assert torch.equal(t1.mem, t2.mem)


def test_nonfinite_score_reports_status(lsa):
    cfg = configs.get("tiny")
    case = cfg.case("cpu")
    g = _to(case)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, 2, 0)
    Q = g["Q"].clone()
    Q[3, 0, 5] = float("nan")
    with pytest.raises(lsa.LsaError) as e:
        lsa.select(tree, Q, g["W"], cfg.beam)
    assert e.value.code == lsa.LSA_ERR_NONFINITE


@pytest.mark.parametrize("G,n_q", [(4, 384), (1, 200), (2, 256), (8, 128)])
def test_tree_attention_matches_oracle(lsa, G, n_q):
    """Leaf-by-leaf tensor-core attention = attention over the expanded key lists."""
    cfg = configs.get("prefill_1m").scaled(n=8 * 8 * 4 * 2 * 64, branching=(8, 8, 4, 2), beam=(4, 16, 16, 8),
                                           Hkv=2, Hq=2 * G, T=n_q, comps=256)
    case = cfg.case("cpu", seed=11 + G)
    g = _to(case)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], leaves=True)
    O, LSE = lsa.tree_attn(tree, g["Q"], g["K"], g["V"], leaves, g["q_pos"], causal=True)
    O2, L2 = lsa.sparse_attn(g["Q"], g["K"], g["V"], idx, g["q_pos"], True)
    torch.cuda.synchronize()
    qp = case.q_pos.numpy()
    for h in range(cfg.Hkv):
        sl = slice(h * G, (h + 1) * G)
        Oo, Lo = orc.attn_fwd(case.Q[:, sl], case.K[h], case.V[h], idx[h].cpu(), q_pos=qp, causal=True)
        mx, mean = parity.attn_errors(O[:, sl].float().cpu(), Oo)
        assert mx <= 2e-2 and mean <= 2e-3, (h, mx, mean)
        assert np.abs(LSE[:, sl].cpu().numpy() - Lo).max() <= 1e-3
    assert (O.float() - O2.float()).abs().max().item() <= 2e-2
    # partial outputs merged in rank order: a second call reproduces every bit
    O3, L3 = lsa.tree_attn(tree, g["Q"], g["K"], g["V"], leaves, g["q_pos"], causal=True)
    assert torch.equal(O, O3) and torch.equal(LSE, L3)


def test_tree_attention_many_queries_per_leaf(lsa):
    """Training geometry, scaled: causal, every leaf chosen by hundreds of queries (several
    128-row chunks per leaf)."""
    cfg = configs.get("train_128k").scaled(n=8192, T=8192, branching=(8, 4, 4), beam=(4, 8, 8), Hkv=2, Hq=8,
                                           comps=64)
    case = cfg.case("cpu")
    g = _to(case)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], leaves=True)
    O, LSE = lsa.tree_attn(tree, g["Q"], g["K"], g["V"], leaves, g["q_pos"], causal=True)
    torch.cuda.synchronize()
    qp = case.q_pos.numpy()
    rows = np.random.default_rng(0).choice(cfg.T, 512, replace=False)
    for h in range(cfg.Hkv):
        sl = slice(h * cfg.G, (h + 1) * cfg.G)
        Oo, Lo = orc.attn_fwd(case.Q[rows][:, sl], case.K[h], case.V[h], idx[h].cpu()[rows], q_pos=qp[rows],
                              causal=True)
        mx, mean = parity.attn_errors(O[rows][:, sl].float().cpu(), Oo)
        assert mx <= 2e-2 and mean <= 2e-3, (h, mx, mean)
        assert np.abs(LSE[rows][:, sl].cpu().numpy() - Lo).max() <= 1e-3


def test_tree_attention_fallback_shapes(lsa):
    """fp32 (tiny workload): the entry point expands the leaves and runs the generic kernels."""
    cfg = configs.get("tiny")
    case = cfg.case("cpu")
    g = _to(case)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select(tree, g["Q"], g["W"], cfg.beam, None, leaves=True)
    O, LSE = lsa.tree_attn(tree, g["Q"], g["K"], g["V"], leaves)
    torch.cuda.synchronize()
    Oo, Lo = orc.attn_fwd(case.Q, case.K[0], case.V[0], idx[0].cpu())
    assert np.abs(O.cpu().numpy() - Oo).max() <= 1e-4


def test_kv_append_writes_rows(lsa):
    for dt in (torch.bfloat16, torch.float32):
        K = torch.randn(3, 50, 128, device=DEV).to(dt)
        V = torch.randn(3, 50, 128, device=DEV).to(dt)
        K0, V0 = K.clone(), V.clone()
        kr = torch.randn(3, 128, device=DEV).to(dt)
        vr = torch.randn(3, 128, device=DEV).to(dt)
        lsa.lsa_kv_append(K, V, 17, kr, vr)
        torch.cuda.synchronize()
        assert torch.equal(K[:, 17], kr) and torch.equal(V[:, 17], vr)
        K[:, 17], V[:, 17] = K0[:, 17], V0[:, 17]
        assert torch.equal(K, K0) and torch.equal(V, V0)
    with pytest.raises(lsa.LsaError):
        lsa.lsa_kv_append(K, V, 50, kr, vr)


@pytest.mark.parametrize("G", [4, 1])
def test_tree_attention_backward(lsa, G):
    """Leaf-by-leaf tensor-core backward = oracle gradient (and = the key-list backward)."""
    cfg = configs.get("train_128k").scaled(n=8192, T=8192, branching=(8, 4, 4), beam=(4, 8, 8), Hkv=2, Hq=2 * G,
                                           comps=64)
    case = cfg.case("cpu", seed=21 + G)
    g = _to(case)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    idx, leaves = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], leaves=True)
    O, LSE = lsa.tree_attn(tree, g["Q"], g["K"], g["V"], leaves, g["q_pos"], causal=True)
    dQ, dK, dV = lsa.tree_attn_bwd(tree, g["Q"], g["K"], g["V"], O, LSE, g["dO"], leaves, g["q_pos"], causal=True)
    dQ2, dK2, dV2 = lsa.sparse_attn_bwd(g["Q"], g["K"], g["V"], O, LSE, g["dO"], idx, g["q_pos"], True)
    torch.cuda.synchronize()
    qp = case.q_pos.numpy()
    for h in range(cfg.Hkv):
        sl = slice(h * G, (h + 1) * G)
        oQ, oK, oV = orc.attn_bwd(case.Q[:, sl], case.K[h], case.V[h], idx[h].cpu(), case.dO[:, sl],
                                  q_pos=qp, causal=True)
        for name, got, want in (("dQ", dQ[:, sl], oQ), ("dK", dK[h], oK), ("dV", dV[h], oV)):
            _check_grad(name, got.cpu().numpy(), want)
    for a, b in ((dQ, dQ2), (dK, dK2), (dV, dV2)):
        ref = b.abs().max().item()
        assert (a - b).abs().max().item() <= 2e-2 * ref


@pytest.mark.parametrize("name,T,Hkv,extra", [
    ("tiny", 1536, 1, {}),
    ("decode_128k", 640, 2, {}),
    ("prefill_1m", 640, 2, dict(n=8 * 8 * 4 * 2 * 64, branching=(8, 8, 4, 2), beam=(4, 16, 16, 8), comps=256)),
])
def test_select_batch_kernels_agree(lsa, name, T, Hkv, extra):
    """A large batch runs the warp-per-query walk, a small one the CTA-per-query walk; both
    sum scores in the same order, so a query's selection must not depend on the batch it
    came in.  The large batch is also checked stage-wise against the oracle."""
    base = configs.get(name)
    cfg = base.scaled(T=T, Hkv=Hkv, Hq=Hkv * (base.Hq // base.Hkv), **extra)
    case = cfg.case("cpu")
    g = _to(case)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    assert T * Hkv >= 148 * 8 and 100 * Hkv < 148 * 8
    idx, qlat, beams = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], qlat=True, beams=True)
    lo, hi = T // 3, T // 3 + 100
    qp = None if g["q_pos"] is None else g["q_pos"][lo:hi].contiguous()
    idx_s, qlat_s = lsa.select(tree, g["Q"][lo:hi].contiguous(), g["W"], cfg.beam, qp, qlat=True)
    torch.cuda.synchronize()
    assert torch.equal(idx[:, lo:hi], idx_s)
    assert torch.equal(qlat[lo:hi], qlat_s)
    qpn = None if case.q_pos is None else case.q_pos.numpy()
    for h in range(Hkv):
        Z = orc.project(case.K[h, :cfg.n], case.W[h])
        th = parity.export_tree(tree, h)
        oq = orc.query_latent(case.Q[:, h * cfg.G:(h + 1) * cfg.G], case.W[h])
        np.testing.assert_allclose(qlat[:, h].cpu().numpy(), oq, rtol=1e-4, atol=1e-5)
        parity.check_select_stagewise(oq, th, cfg.branching, cfg.leaf, cfg.beam, qpn,
                                      beams[:, h].cpu().numpy(), idx[h].cpu().numpy())
