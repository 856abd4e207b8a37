"""Partitioning the SSA hot path over ranks (host logic only).

Each (batch, kv head) group is independent: its block selection, both
attention streams, the dropped mass and the backward need only the g query
heads that read that kv head.  A problem is split over ranks by kv-head
ranges; each rank passes strided views of its heads to the C ABI (no copies).

The alignment loss is a mean over all B*Hq*N*d elements, so a shard that holds
M_local of the M_global elements must scale alpha by M_local / M_global for
its per-element gradient 2*alpha*(h_f - h_s)/M to match the unsharded
objective, and the global loss is the M-weighted sum of the shard losses --
one scalar all-reduce, the only exchange the path has.
"""
from __future__ import annotations


def kv_head_range(Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous kv heads [lo, hi) of `rank`; sizes differ by at most one."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    base, extra = divmod(Hkv, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def shard_views(Q, K, V, group: int, lo: int, hi: int):
    """Views of one rank's heads: Q[:, lo*g:hi*g], K[:, lo:hi], V[:, lo:hi]."""
    return Q[:, lo * group:hi * group], K[:, lo:hi], V[:, lo:hi]


def local_alpha(alpha: float, m_local: int, m_global: int) -> float:
    return float(alpha) * m_local / m_global


def combine_align_loss(local_loss: float, m_local: int, m_global: int, all_reduce_sum) -> float:
    """Global L_align from a shard's L_align; `all_reduce_sum` sums a float over ranks."""
    return all_reduce_sum(local_loss * m_local / m_global)
