"""The decode step (lsa_decode_step: append, select, attention in two launches) through the
C ABI, against the separate calls (lsa_select, lsa_sparse_attn) and against the oracle.

Each step appends the token's key and value rows, keeps beam[-1] leaves per KV group and
attends to their keys plus the dense tail of appended rows, causal by position.  Shapes
cover bf16 and fp32, d = 64 and 128, 1 to 8 query heads per group, leaves of 16, 64 and 128
keys (one or two 64-key splits per leaf), an empty tail, and replays of a captured graph
(the split counters re-arm themselves).
"""
import math

import numpy as np
import pytest
import torch

from hierarchical_latent_key_b200 import configs
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = {
    "decode_128k_2heads": lambda: configs.get("decode_128k").scaled(Hkv=2, Hq=8, T=12),
    "tiny_f32": lambda: configs.get("tiny").scaled(T=10, mode="decode"),
    "bf16_d64_G8_leaf128": lambda: configs.get("decode_128k").scaled(
        name="g8", n=16 * 8 * 128, branching=(16, 8), beam=(4, 6), leaf=128, Hkv=1, Hq=8, d=64, r=32, T=9, comps=64),
    "bf16_G2": lambda: configs.get("decode_128k").scaled(n=16 * 16 * 64, branching=(16, 16), beam=(8, 16), Hkv=3,
                                                          Hq=6, T=7, comps=128),
}


@pytest.fixture(scope="module")
def lsa():
    from hierarchical_latent_key_b200 import lsa as mod
    return mod


def _tol(cfg):
    return (1e-4, 1e-4) if cfg.dtype == "f32" else (2e-2, 2e-3)


@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_step_matches_calls_and_oracle(lsa, name):
    cfg = CASES[name]()
    case = cfg.case(DEV)
    n = cfg.n
    Knew = case.K[:, n:].transpose(0, 1).clone(memory_format=torch.contiguous_format)
    Vnew = case.V[:, n:].transpose(0, 1).clone(memory_format=torch.contiguous_format)
    K0, V0 = case.K.clone(), case.V.clone()       # reference caches, rows present from the start
    case.K[:, n:].zero_()
    case.V[:, n:].zero_()
    tree = lsa.build_tree(case.K, case.W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    dec = lsa.DecodeStep(tree, case.W, cfg.beam, case.K, cfg.Hq, cfg.T)
    tmax, tmean = _tol(cfg)
    li = tree.leaf_index().cpu().numpy()
    for s in range(cfg.T):
        pos = n + s
        Qs = case.Q[s:s + 1]
        O, LSE = dec.step(case.K, case.V, Qs, Knew[s], Vnew[s], pos, n)
        torch.cuda.synchronize()
        assert lsa.lsa_status_check(dec.status) == lsa.LSA_OK
        # appended rows
        assert torch.equal(case.K[:, pos], K0[:, pos]) and torch.equal(case.V[:, pos], V0[:, pos])
        # the same selection as the select call
        idx, leaves = lsa.select(tree, Qs, case.W, cfg.beam, torch.tensor([pos], dtype=torch.int32, device=DEV),
                                 leaves=True)
        assert torch.equal(dec.leaves, leaves[:, 0])
        # the separate attention call on the same keys
        O2, L2 = lsa.sparse_attn(Qs, K0, V0, idx, torch.tensor([pos], dtype=torch.int32, device=DEV), True,
                                 (n, pos + 1))
        d = (O.float() - O2.float()).abs()
        assert d.max().item() <= tmax and d.mean().item() <= tmean, (s, d.max().item())
        assert (LSE - L2).abs().max().item() <= 1e-3
        # the oracle on the kept leaves' keys and the tail
        for h in range(cfg.Hkv):
            kept = dec.leaves[h].cpu().numpy()
            keys = np.concatenate([li[h].reshape(-1, cfg.leaf)[k] for k in kept if k >= 0] +
                                  [np.arange(n, pos + 1)])
            sl = slice(h * cfg.G, (h + 1) * cfg.G)
            Kc = K0[h, torch.as_tensor(keys, device=DEV)].double().cpu().numpy()
            Vc = V0[h, torch.as_tensor(keys, device=DEV)].double().cpu().numpy()
            Oo, Lo = orc.attn_fwd(Qs[:, sl].double().cpu().numpy(), Kc, Vc,
                                  np.zeros((1, 0), np.int32), tail=(0, len(keys)))
            mx, mean = parity.attn_errors(O[:, sl].float().cpu(), Oo)
            assert mx <= tmax and mean <= tmean, (s, h, mx, mean)
            assert np.abs(LSE[:, sl].cpu().numpy() - Lo).max() <= 1e-3


def test_decode_step_empty_tail_and_graph_replay(lsa):
    cfg = CASES["decode_128k_2heads"]()
    case = cfg.case(DEV)
    n = cfg.n
    tree = lsa.build_tree(case.K, case.W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    dec = lsa.DecodeStep(tree, case.W, cfg.beam, case.K, cfg.Hq, 4)
    # pos = n - 1: the token is the last indexed key; tail [n, n) is empty, no append
    O, LSE = dec.step(case.K, case.V, case.Q[:1], None, None, n - 1, n)
    O1, L1 = O.clone(), LSE.clone()
    idx = lsa.select(tree, case.Q[:1], case.W, cfg.beam, torch.tensor([n - 1], dtype=torch.int32, device=DEV))
    O2, L2 = lsa.sparse_attn(case.Q[:1], case.K, case.V, idx, torch.tensor([n - 1], dtype=torch.int32, device=DEV),
                             True)
    assert (O1.float() - O2.float()).abs().max().item() <= 2e-2
    # a captured step replayed: every replay re-arms the split counters and gives the same output
    Kr, Vr = case.K[:, n + 1].contiguous(), case.V[:, n + 1].contiguous()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        dec.step(case.K, case.V, case.Q[1:2], Kr, Vr, n + 1, n, stream=st)
    torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    want = dec.O.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        dec.step(case.K, case.V, case.Q[1:2], Kr, Vr, n + 1, n, stream=st)
    for _ in range(3):
        dec.O.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(dec.O, want)
    assert lsa.lsa_status_check(dec.status) == lsa.LSA_OK
