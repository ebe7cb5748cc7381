"""The batched schedule of the hierarchical search (lsa_select_batched) against the
walk-by-walk one (lsa_select) and the oracle.

Both compute every score with the same fp32 expression and rank with the same code,
so their outputs must agree exactly; the prefill-shaped case is also checked
stage-wise against the oracle (near-tie band as for lsa_select)."""
import numpy as np
import pytest
import torch

from hierarchical_latent_key_b200 import configs
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from hierarchical_latent_key_b200 import lsa as mod
    return mod


def _to(case):
    return {k: (None if v is None else v.to(DEV)) for k, v in
            dict(K=case.K, V=case.V, W=case.W, Q=case.Q, q_pos=case.q_pos).items()}


CASES = [
    ("tiny", dict(T=1536)),
    ("tiny", dict(T=3)),
    ("decode_128k", dict(T=637, Hkv=2, Hq=8)),
    ("prefill_1m", dict(T=645, Hkv=2, Hq=8, n=8 * 8 * 4 * 2 * 64, branching=(8, 8, 4, 2), beam=(4, 16, 16, 8),
                        comps=256)),
    ("prefill_1m", dict(T=300, Hkv=2, Hq=4, n=16 * 16 * 4 * 64, branching=(16, 16, 4), beam=(8, 32, 32),
                        comps=256)),
    ("train_128k", dict(T=4096, n=4096, Hkv=2, Hq=8, branching=(8, 4, 2), beam=(4, 8, 8), comps=64)),
]


@pytest.mark.parametrize("name,extra", CASES)
def test_batched_equals_walk_by_walk(lsa, name, extra):
    cfg = configs.get(name).scaled(**extra)
    case = cfg.case("cpu")
    g = _to(case)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    ref = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], qlat=True, beams=True, leaves=True)
    got = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], qlat=True, beams=True, leaves=True, batched=True)
    torch.cuda.synchronize()
    for what, a, b in zip(("idx", "leaves", "qlat", "beams"), got, ref):
        assert torch.equal(a, b), what
    if name == "prefill_1m":
        idx, leaves, qlat, beams = got
        qpn = case.q_pos.numpy()
        near = 0
        for h in range(cfg.Hkv):
            th = parity.export_tree(tree, h)
            oq = orc.query_latent(case.Q[:, h * cfg.G:(h + 1) * cfg.G], case.W[h])
            np.testing.assert_allclose(qlat[:, h].cpu().numpy(), oq, rtol=1e-4, atol=1e-5)
            near += parity.check_select_stagewise(oq, th, cfg.branching, cfg.leaf, cfg.beam, qpn,
                                                  beams[:, h].cpu().numpy(), idx[h].cpu().numpy())
        assert near <= max(2, cfg.T * cfg.Hkv // 100)


def test_batched_causal_prefix_leaves_pads(lsa):
    """Queries at the start of the sequence see few nodes: kept lists shorter than the beam
    are padded with -1 identically on both schedules."""
    cfg = configs.get("prefill_1m").scaled(T=256, Hkv=2, Hq=8, n=8 * 8 * 4 * 2 * 64, branching=(8, 8, 4, 2),
                                           beam=(4, 16, 16, 8), comps=256)
    case = cfg.case("cpu")
    g = _to(case)
    g["q_pos"] = torch.arange(0, 4 * cfg.T, 4, dtype=torch.int32, device=DEV)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    ref = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], beams=True, leaves=True)
    got = lsa.select(tree, g["Q"], g["W"], cfg.beam, g["q_pos"], beams=True, leaves=True, batched=True)
    torch.cuda.synchronize()
    assert (ref[1] < 0).any(), "the case should have queries with fewer eligible leaves than the beam"
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_batched_nonfinite_and_workspace(lsa):
    cfg = configs.get("tiny")
    case = cfg.case("cpu")
    g = _to(case)
    tree = lsa.build_tree(g["K"], g["W"], cfg.branching, cfg.leaf, 2, 0)
    Q = g["Q"].clone()
    Q[3, 0, 5] = float("nan")
    with pytest.raises(lsa.LsaError) as e:
        lsa.select(tree, Q, g["W"], cfg.beam, batched=True)
    assert e.value.code == lsa.LSA_ERR_NONFINITE
    T = g["Q"].shape[0]
    need = lsa.lsa_select_batched_workspace_bytes(tree.desc, T, cfg.beam)
    assert need > 0 and lsa.lsa_select_batched_workspace_bytes(tree.desc, 0, cfg.beam) == 0
    idx = torch.empty(1, T, cfg.beam[-1] * cfg.leaf, dtype=torch.int32, device=DEV)
    small = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_select_batched(tree.desc, tree.mem, g["Q"], g["W"], cfg.beam, None, idx, workspace=small)
    assert e.value.code == lsa.LSA_ERR_WORKSPACE
    # no queries: nothing to do, no workspace needed
    lsa.lsa_select_batched(tree.desc, tree.mem, g["Q"][:0], g["W"], cfg.beam, None, idx[:, :0])
