"""The balanced k-means assignment step through the C ABI (lsa_balanced_assign).

(a) Parity: the GPU's assignment equals the oracle's unique stable balanced assignment
    (pair order: squared distance, row, centroid), or differs only where it stays stable
    within the build's epsilon (fp32 vs fp64 distances), on segments handled by one CTA
    each and on segments large enough for the cooperative grid kernel.
(b) Failure detection without a fault: a proposal-round cap of 1 on inputs that need many
    rounds (every row prefers centroid 0) makes the kernels leave their loop, report
    LSA_ERR_TIMEOUT in the status word and return; the next call on the same context runs
    normally.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def lsa():
    from hierarchical_latent_key_b200 import lsa as mod
    return mod


def _case(nseg, m, b, r, seed, crowd=False):
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((nseg * m, r)).astype(np.float32)
    mu = np.empty((nseg * b, r), np.float32)
    for s in range(nseg):
        Zs = Z[s * m:(s + 1) * m]
        mu[s * b:(s + 1) * b] = Zs[rng.choice(m, b, replace=False)]
        if crowd:   # centroid 0 at the segment mean, the others far away: every row prefers 0
            mu[s * b] = Zs.mean(axis=0)
            mu[s * b + 1:(s + 1) * b] += 6.0
    return Z, mu


@pytest.mark.parametrize("nseg,m,b,r", [(37, 64, 4, 16), (5, 4096, 16, 64), (3, 1000, 8, 32),
                                        (2, 65536, 8, 64), (1, 20000, 5, 64)])
def test_assign_matches_oracle(lsa, nseg, m, b, r):
    Z, mu = _case(nseg, m, b, r, seed=nseg * m + b)
    choice = lsa.balanced_assign(torch.from_numpy(Z).to(DEV), torch.from_numpy(mu).to(DEV), nseg, m, b)
    got = choice.cpu().numpy().astype(np.int64)
    differing = 0
    pos = np.arange(m)
    for s in range(nseg):
        Zs = Z[s * m:(s + 1) * m].astype(np.float64)
        ms = mu[s * b:(s + 1) * b].astype(np.float64)
        D = orc.distances(Zs, ms)
        want = orc.balanced_assign(D, pos)
        g = got[s * m:(s + 1) * m]
        assert np.all(np.bincount(g, minlength=b) == m // b), s
        if not np.array_equal(g, want):
            assert parity._eps_stable(D, g, Zs, ms), s
            differing += 1
    assert differing <= max(1, nseg // 10), differing


@pytest.mark.parametrize("nseg,m,b", [(16, 512, 8), (2, 32768, 8)])
def test_round_cap_reports_timeout_and_returns(lsa, nseg, m, b):
    Z, mu = _case(nseg, m, b, 64, seed=3, crowd=True)
    Zd, mud = torch.from_numpy(Z).to(DEV), torch.from_numpy(mu).to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    lsa.balanced_assign(Zd, mud, nseg, m, b, max_rounds=1, status=st, check=False)
    assert lsa.lsa_status_check(st) == lsa.LSA_ERR_TIMEOUT
    # the context is still usable: the same inputs without the cap give the balanced answer
    st.zero_()
    choice = lsa.balanced_assign(Zd, mud, nseg, m, b, status=st, check=False)
    assert lsa.lsa_status_check(st) == lsa.LSA_OK
    got = choice.cpu().numpy().astype(np.int64).reshape(nseg, m)
    for s in range(nseg):
        assert np.all(np.bincount(got[s], minlength=b) == m // b)
