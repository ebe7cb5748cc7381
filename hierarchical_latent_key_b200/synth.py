"""Seeded synthetic inputs for the LSA hot path.

This module holds no arithmetic of the method itself: it only draws the
workload tensors (queries, keys, values, latent projection, upstream gradient)
from seeded generators.  Both the CUDA path and the CPU oracle consume exactly
the tensors it returns, so it is the one module the two sides share.

Recipe (per KV head h, for every workload):
  * mixture centres: ``comps`` vectors N(0, I_d), each normalised to unit norm;
  * key at position p: a component drawn uniformly, plus N(0, sigma^2 I) noise,
    sigma = 0.3 (components are i.i.d. over positions: no positional locality);
  * value rows: N(0, I_d);
  * latent projection W[h]: [d, r] with entries N(0, 1/d);
  * query of token t for GQA group g: one component of head g's mixture drawn
    uniformly; each of the G query heads of the group is that centre plus
    N(0, sigma^2 I) noise;
  * upstream gradient (training workload): N(0, I_d) per query head;
  * bf16 tensors are the float32 draws rounded to nearest even.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

SIGMA = 0.3
_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _DT[name]


@dataclass
class Case:
    """One workload's tensors.  Shapes:
    Q [T, Hq, d]; K, V [Hkv, n_cap, d]; W [Hkv, d, r]; q_pos [T] int32 or None;
    dO [T, Hq, d] or None.  The tree covers positions [0, n); positions
    [n, n_cap) are appended during decode."""
    Q: torch.Tensor
    K: torch.Tensor
    V: torch.Tensor
    W: torch.Tensor
    q_pos: torch.Tensor | None
    dO: torch.Tensor | None
    n: int
    n_cap: int
    comp_of_query: torch.Tensor | None = None


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def mixture_centres(g, Hkv: int, comps: int, d: int, device) -> torch.Tensor:
    c = torch.randn(Hkv, comps, d, generator=g, device=device, dtype=torch.float32)
    return c / c.norm(dim=-1, keepdim=True)


def mixture_rows(g, centres: torch.Tensor, rows: int, dtype, device, chunk: int = 1 << 20,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """[Hkv, rows, d] draws from each head's mixture (chunked to bound fp32 scratch)."""
    Hkv, comps, d = centres.shape
    if out is None:
        out = torch.empty(Hkv, rows, d, dtype=dtype, device=device)
    for h in range(Hkv):
        for s in range(0, rows, chunk):
            e = min(rows, s + chunk)
            comp = torch.randint(0, comps, (e - s,), generator=g, device=device)
            x = centres[h, comp] + SIGMA * torch.randn(e - s, d, generator=g, device=device)
            out[h, s:e] = x.to(dtype)
    return out


def normal_rows(g, shape, dtype, device, chunk_rows: int = 1 << 20, out=None) -> torch.Tensor:
    """N(0,1) tensor of `shape` (last dim = row), drawn in chunks of rows."""
    if out is None:
        out = torch.empty(*shape, dtype=dtype, device=device)
    flat = out.view(-1, shape[-1])
    for s in range(0, flat.shape[0], chunk_rows):
        e = min(flat.shape[0], s + chunk_rows)
        flat[s:e] = torch.randn(e - s, shape[-1], generator=g, device=device).to(dtype)
    return out


def make_case(*, n: int, n_cap: int, T: int, Hq: int, Hkv: int, d: int, r: int, comps: int,
              dtype: str, seed: int, q_pos=None, with_grad: bool = False,
              device="cpu") -> Case:
    """Draw one workload.  q_pos: None (non-causal) or an int32 tensor/list of T positions."""
    dt = torch_dtype(dtype)
    g = _gen(seed, device)
    G = Hq // Hkv
    centres = mixture_centres(g, Hkv, comps, d, device)
    K = mixture_rows(g, centres, n_cap, dt, device)
    V = normal_rows(g, (Hkv, n_cap, d), dt, device)
    W = (torch.randn(Hkv, d, r, generator=g, device=device) / d ** 0.5).to(dt)
    comp = torch.randint(0, comps, (T, Hkv), generator=g, device=device)
    base = centres[torch.arange(Hkv, device=device)[None, :], comp]          # [T, Hkv, d]
    noise = SIGMA * torch.randn(T, Hkv, G, d, generator=g, device=device)
    Q = (base[:, :, None, :] + noise).reshape(T, Hq, d).to(dt)
    dO = normal_rows(g, (T, Hq, d), dt, device) if with_grad else None
    if q_pos is not None and not isinstance(q_pos, torch.Tensor):
        q_pos = torch.tensor(q_pos, dtype=torch.int32, device=device)
    return Case(Q=Q, K=K, V=V, W=W, q_pos=q_pos, dO=dO, n=n, n_cap=n_cap, comp_of_query=comp)
