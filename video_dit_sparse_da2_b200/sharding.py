"""Multi-GPU decomposition of one call: (batch, head) units are independent
problems -- the draft map, the per-head ranking and quotas, and the value
units sigma are all per head ("DraftAttention2", Sec. 3.1 "Joint allocation
of sparsity and precision": ranking within each head) -- so a call splits
across ranks by heads with no data exchange; each rank runs the path on its
heads and writes its slice of the output."""
from __future__ import annotations


def head_shard(n_units: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous range [lo, hi) of units (flattened batch x head) of `rank`:
    balanced, the first n_units % world ranks take one more."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)
