"""The five workloads of the LSA hot path, with their tree and search parameters.

Names and sizes:
  tiny          fp32, 1 KV head, d=64, r=16, n=4096 keys; tree 16 x 16, leaf 16;
                beam 4 top nodes then 8 leaves (128 keys); 256 queries, non-causal.
  decode_128k   bf16, 32 query / 8 KV heads, d=128, r=64, n=131072; tree 16/256/2048
                nodes, leaf 64; beam 8/32/32 (2048 keys); 256 single-token decode
                steps, each appending one key that joins a dense tail.
  prefill_1m    bf16, 32/8 heads, n=1,048,576 cached keys; tree 16,16,16,4, leaf 64;
                beam 8/32/32/32 (2048 keys); the last 4096 positions are the query
                chunk (causal by position).
  decode_10m    bf16, 32/8 heads, n=10,485,760; tree 8,16,16,16,5, leaf 64 (163840
                leaves); beam 8/16/32/32/32 (2048 keys); 128 decode steps.
  train_128k    bf16, 16/4 heads, n=T=131072, causal; tree 16,16,8, leaf 64; beam
                8/32/32 (2048 keys); tree rebuilt each step; forward + backward.

Where the workload statements leave a parameter open (k-means iterations and seeds
beyond the tiny case, the prefill beam per level, the training tree), the values
below are the readings used.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

from . import synth


@dataclass(frozen=True)
class Config:
    name: str
    dtype: str
    n: int            # keys covered by the tree
    Hq: int
    Hkv: int
    d: int
    r: int
    branching: tuple
    leaf: int
    beam: tuple
    T: int            # queries (batch / chunk / decode steps)
    comps: int        # mixture components per KV head
    iters: int        # balanced k-means iterations per level
    mode: str         # "batch" | "decode" | "prefill" | "train"
    seed: int
    rebuild_every: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def K_sel(self) -> int:
        return self.beam[-1] * self.leaf

    @property
    def causal(self) -> bool:
        return self.mode in ("decode", "prefill", "train")

    @property
    def n_cap(self) -> int:
        return self.n + (self.T if self.mode == "decode" else 0)

    @property
    def nodes(self) -> list:
        return [int(x) for x in np.cumprod(self.branching)]

    def q_pos(self):
        if self.mode == "batch":
            return None
        if self.mode == "decode":
            return [self.n + s for s in range(self.T)]
        if self.mode == "prefill":
            return [self.n - self.T + i for i in range(self.T)]
        return list(range(self.T))

    def check(self):
        assert int(np.prod(self.branching)) * self.leaf == self.n, self.name
        assert self.Hq % self.Hkv == 0
        avail = self.nodes[0]
        for l, b in enumerate(self.beam):
            assert 1 <= b <= avail, (self.name, l)
            if l + 1 < len(self.beam):
                avail = b * self.branching[l + 1]
        return self

    def case(self, device="cpu", seed=None):
        return synth.make_case(n=self.n, n_cap=self.n_cap, T=self.T, Hq=self.Hq, Hkv=self.Hkv,
                               d=self.d, r=self.r, comps=self.comps, dtype=self.dtype,
                               seed=self.seed if seed is None else seed, q_pos=self.q_pos(),
                               with_grad=self.mode == "train", device=device)

    def scaled(self, **kw) -> "Config":
        return replace(self, **kw).check()


CONFIGS = {
    "tiny": Config("tiny", "f32", 4096, 1, 1, 64, 16, (16, 16), 16, (4, 8), 256, 32, 10,
                   "batch", 0),
    "decode_128k": Config("decode_128k", "bf16", 131072, 32, 8, 128, 64, (16, 16, 8), 64,
                          (8, 32, 32), 256, 1024, 10, "decode", 1, rebuild_every=4096),
    "prefill_1m": Config("prefill_1m", "bf16", 1 << 20, 32, 8, 128, 64, (16, 16, 16, 4), 64,
                         (8, 32, 32, 32), 4096, 8192, 10, "prefill", 2),
    "decode_10m": Config("decode_10m", "bf16", 10485760, 32, 8, 128, 64, (8, 16, 16, 16, 5), 64,
                         (8, 16, 32, 32, 32), 128, 65536, 10, "decode", 3, rebuild_every=4096),
    "train_128k": Config("train_128k", "bf16", 131072, 16, 4, 128, 64, (16, 16, 8), 64,
                         (8, 32, 32), 131072, 1024, 10, "train", 4),
}
for _c in CONFIGS.values():
    _c.check()


def get(name: str) -> Config:
    return CONFIGS[name]
