"""Host-side sharding of independent (sequence, head) recurrences across ranks.

Every (sequence, head) pair of KDA is an independent recurrence, so a batch
splits across GPUs with no exchange on the data path: rank r takes a
contiguous block of sequences.  Only the timing uses a collective (the max
over ranks).  Used by bench.py; tested with the gloo backend on CPU.
"""
from __future__ import annotations


def shard_bounds(n_units: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, stop) block of n_units for this rank; sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world or n_units < 0:
        raise ValueError("need 0 <= rank < world and n_units >= 0")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(values, group=None, device=None):
    """Element-wise max of a list of floats over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t.tolist()
