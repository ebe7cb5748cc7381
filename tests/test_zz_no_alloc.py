"""The allocation-free attention entry point (GPU).

Some callers cannot allocate device memory: a plugin whose host framework hands it only
its input and output buffers, or a serving loop that must not call cudaMalloc once it has
started (the call can synchronise the whole device).  They use lsa_sparse_attn_noalloc,
whose split partials live in a built-in device array instead of a caller workspace.  Its
results must match lsa_sparse_attn on the same inputs, also when the array still holds
an earlier call's partials.
"""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def lsa():
    from hierarchical_latent_key_b200 import lsa as mod
    return mod


def _case(seed, T, Hkv, G, d, n_cap, K_sel, dtype, tail):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(T, Hkv * G, d, generator=g).to(dtype)
    K = torch.randn(Hkv, n_cap, d, generator=g).to(dtype)
    V = torch.randn(Hkv, n_cap, d, generator=g).to(dtype)
    idx = torch.stack([torch.stack([torch.randperm(tail[0], generator=g)[:K_sel] for _ in range(T)])
                       for _ in range(Hkv)]).int()
    idx[:, :, -5:] = -1
    q_pos = torch.full((T,), tail[1] - 1, dtype=torch.int32) - torch.arange(T, dtype=torch.int32)
    return [x.to(DEV) for x in (Q, K, V, idx, q_pos)]


CASES = [  # decode-shaped (split over many CTAs, uses the built-in scratch), then a small one
    dict(seed=1, T=1, Hkv=8, G=4, d=128, n_cap=140000, K_sel=2048, dtype=torch.bfloat16, tail=(131072, 131172),
         causal=True),
    dict(seed=2, T=3, Hkv=2, G=4, d=64, n_cap=5000, K_sel=203, dtype=torch.float32, tail=(4000, 4077),
         causal=False),
]


def test_noalloc_matches_workspace_entry_point(lsa):
    for rep in range(2):                 # the second pass finds the previous call's partials
        for c in CASES:
            Q, K, V, idx, q_pos = _case(c["seed"] + rep, c["T"], c["Hkv"], c["G"], c["d"], c["n_cap"],
                                        c["K_sel"], c["dtype"], c["tail"])
            scale = 1.0 / math.sqrt(c["d"])
            need = lsa.lsa_attn_workspace_bytes(c["T"], c["Hkv"] * c["G"], c["Hkv"], c["d"], c["K_sel"],
                                                c["tail"][1] - c["tail"][0])
            if c["T"] == 1:
                assert need > 0        # this case exercises the built-in scratch
            O_ref, L_ref = lsa.sparse_attn(Q, K, V, idx, q_pos, c["causal"], c["tail"], scale)
            O = torch.empty_like(Q)
            LSE = torch.empty(c["T"], c["Hkv"] * c["G"], dtype=torch.float32, device=DEV)
            status = torch.zeros(1, dtype=torch.int32, device=DEV)
            lsa.lsa_sparse_attn_noalloc(Q, K, V, idx, q_pos, c["causal"], c["tail"][0], c["tail"][1], scale, O,
                                        LSE, status)
            assert lsa.lsa_status_check(status) == 0
            tmax, tmean = (1e-4, 1e-4) if c["dtype"] == torch.float32 else (2e-2, 2e-3)
            err = (O.float() - O_ref.float()).abs()
            assert err.max().item() <= tmax and err.mean().item() <= tmean
            assert torch.allclose(LSE, L_ref, atol=1e-3, rtol=0)


def test_noalloc_rejects_requests_beyond_the_array(lsa):
    T, Hkv, G, d, K_sel = 591, 1, 8, 128, 128    # 2 splits x 591 queries x 8 heads: ~4.9 MB of partials
    Q = torch.zeros(T, Hkv * G, d, dtype=torch.bfloat16, device=DEV)
    K = torch.zeros(Hkv, 1024, d, dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros(Hkv, T, K_sel, dtype=torch.int32, device=DEV)
    O = torch.empty_like(Q)
    LSE = torch.empty(T, Hkv * G, dtype=torch.float32, device=DEV)
    assert lsa.lsa_attn_workspace_bytes(T, Hkv * G, Hkv, d, K_sel, 0) > (4 << 20)
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_sparse_attn_noalloc(Q, K, K, idx, None, False, 0, 0, 0.1, O, LSE)
    assert e.value.code == lsa.LSA_ERR_WORKSPACE
    assert "built-in array" in str(e.value)
