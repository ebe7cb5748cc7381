"""Latent projection Z = K . W through the C ABI (lsa_project_keys) against fp64 products.

bf16 inputs run on the tensor cores: every product of two bf16 values is exact in fp32
and only the fp32 summation order differs from the fp64 sum, so each element must lie
within 8 d u32 of the sum of |products| (u32 = 2^-24; sum of d rounded additions).  fp32
inputs (fp32 FMAs) get the same bound.  Sizes span several 128-key tiles with a ragged
last tile, every supported (d, r) pair, and a full-size head of the 1M-key prefill.
"""
import numpy as np
import pytest
import torch

from hierarchical_latent_key_b200 import configs

pytestmark = pytest.mark.gpu
DEV = "cuda"
U32 = 2.0 ** -24


@pytest.fixture(scope="module")
def lsa():
    from hierarchical_latent_key_b200 import lsa as mod
    return mod


def _check(Z, K, W, n, rows=None):
    Kd = K[:, :n].double().cpu().numpy()
    Wd = W.double().cpu().numpy()
    Zg = Z.double().cpu().numpy()
    for h in range(K.shape[0]):
        k = Kd[h] if rows is None else Kd[h][rows]
        z = Zg[h] if rows is None else Zg[h][rows]
        ref = k @ Wd[h]
        mag = np.abs(k) @ np.abs(Wd[h])
        bound = 8 * K.shape[2] * U32 * mag + 1e-30
        assert np.all(np.abs(z - ref) <= bound), (h, float((np.abs(z - ref) / bound).max()))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,r", [(128, 64), (128, 32), (128, 16), (64, 64), (64, 32), (64, 16)])
def test_project_matches_fp64(lsa, dtype, d, r):
    torch.manual_seed(d * 7 + r)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    H, n_cap, n = 3, 5000, 4871          # 38 full tiles + a ragged one per head; rows past n untouched
    K = torch.randn(H, n_cap, d).to(dt).to(DEV)
    W = (torch.randn(H, d, r) / d ** 0.5).to(dt).to(DEV)
    Z = torch.full((H, n, r), float("nan"), dtype=torch.float32, device=DEV)
    lsa.lsa_project_keys(K, W, n, Z)
    torch.cuda.synchronize()
    assert torch.isfinite(Z).all()
    _check(Z, K, W, n)


def test_project_empty_and_single(lsa):
    K = torch.randn(2, 300, 128, dtype=torch.bfloat16, device=DEV)
    W = torch.randn(2, 128, 64, dtype=torch.bfloat16, device=DEV)
    Z = torch.empty(2, 0, 64, dtype=torch.float32, device=DEV)
    lsa.lsa_project_keys(K, W, 0, Z)
    Z1 = lsa.project_keys(K, W, 1)
    torch.cuda.synchronize()
    _check(Z1, K, W, 1)


def test_project_prefill_head_full_size(lsa):
    """All 8 heads of the 1,048,576-key prefill index (the launch the build makes), 4096
    sampled keys per head checked."""
    cfg = configs.get("prefill_1m")
    torch.manual_seed(5)
    K = torch.randn(cfg.Hkv, cfg.n, 128, device=DEV).to(torch.bfloat16)
    W = (torch.randn(cfg.Hkv, 128, cfg.r, device=DEV) / 128 ** 0.5).to(torch.bfloat16)
    Z = lsa.project_keys(K, W)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(cfg.n, 4096, replace=False))
    _check(Z, K, W, cfg.n, rows=rows)
