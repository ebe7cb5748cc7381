"""Host logic of a KV-head split: one request served by several ranks, no exchange inside
the layer.

The index, the selection and the attention of a KV head depend only on that head's keys,
values and the queries of its GQA group, so a request's KV heads can be spread over ranks
(one process per GPU): rank r owns the contiguous KV heads ``head_range(r, world, Hkv)``
and the query heads of their groups, builds and searches its own index over them, and
produces those query heads' outputs.  The only communication is gathering the per-rank
output slices into [T, Hq, d] where a caller needs the whole layer output on one rank.
"""
from __future__ import annotations

import torch


def head_range(rank: int, world: int, n_kv_heads: int) -> tuple[int, int]:
    """Contiguous KV heads [lo, hi) of `rank`; the first n_kv_heads % world ranks get one more."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    base, extra = divmod(n_kv_heads, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def query_range(kv_lo: int, kv_hi: int, group: int) -> tuple[int, int]:
    """Query heads of the GQA groups of KV heads [kv_lo, kv_hi) (query head h is in group h // G)."""
    return kv_lo * group, kv_hi * group


def local_inputs(Q, K, V, W, rank: int, world: int):
    """The rank's slices of one request: Q [T, Hq_r, d], K/V [Hkv_r, n_cap, d], W [Hkv_r, d, r]
    (contiguous copies, as the C ABI takes dense tensors)."""
    Hkv = K.shape[0]
    G = Q.shape[1] // Hkv
    lo, hi = head_range(rank, world, Hkv)
    qlo, qhi = query_range(lo, hi, G)
    return (Q[:, qlo:qhi].contiguous(), K[lo:hi].contiguous(), V[lo:hi].contiguous(), W[lo:hi].contiguous())


def stitch_heads(parts):
    """Per-rank outputs [T, Hq_r, ...] in rank order -> [T, Hq, ...]."""
    return torch.cat(list(parts), dim=1)


def gather_heads(local, world: int, n_kv_heads: int, group=None):
    """All-gather of every rank's output slice [T, Hq_r, ...] into [T, Hq, ...] on every rank.
    Slices may differ in head count (uneven splits): each is padded to the largest before
    the collective and trimmed after it."""
    import torch.distributed as dist

    G_heads = [hi - lo for lo, hi in (head_range(r, world, n_kv_heads) for r in range(world))]
    per_kv = local.shape[1] // max(1, G_heads[dist.get_rank(group)])
    widest = max(G_heads) * per_kv
    pad = torch.zeros((local.shape[0], widest) + tuple(local.shape[2:]), dtype=local.dtype, device=local.device)
    pad[:, :local.shape[1]] = local
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad, group=group)
    return stitch_heads(b[:, :n * per_kv] for b, n in zip(bufs, G_heads))
