"""Row sharding across ranks (one process per GPU).

Rows of a verification batch are independent and the uniforms are keyed by
the global row id (Philox counter), so a batch splits across ranks with no
data-path collective: rank r verifies a contiguous block of rows with
`row_base` set to the block's first global row, and the concatenated
outputs equal the unsharded result.  The only collectives are the timing
barrier and the max-over-ranks reduction of the measured time.
"""
from __future__ import annotations

import torch


def shard_rows(total_rows: int, world: int, rank: int):
    """Contiguous block [start, stop) of rank `rank`; sizes differ by at most 1."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(total_rows, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
