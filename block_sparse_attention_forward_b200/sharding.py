"""Head sharding across ranks.

Every (batch, head) pair of the block-sparse forward is independent: its mask,
CRM rows, token permutation and softmax never look at another head.  So the
path shards by flat head index bh = b*H + h with no exchange between ranks;
a caller that wants every head on one device gathers the outputs afterwards.
"""
from __future__ import annotations


def head_range(n_heads_total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [lo, hi) slice of flat head ids owned by `rank` (balanced to +-1)."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad world/rank")
    base, extra = divmod(n_heads_total, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi
