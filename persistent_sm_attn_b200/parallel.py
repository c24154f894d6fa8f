"""Multi-GPU plumbing for the backward: one process per GPU.

Heads (b, h) are independent in the attention backward (no dQ, dK or dV
crosses heads), so a batch of B*H heads is split into contiguous per-rank
ranges and every rank runs the deterministic kernel on its own range with no
data-path collective.  The results of a head do not depend on how many ranks
share the batch.  The only communication is timing: the max over ranks.
"""
from __future__ import annotations


def head_range(n_heads: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, end) range of flattened heads owned by `rank`.

    The first n_heads % world ranks get one extra head, so ranges differ in
    size by at most one and together cover 0..n_heads-1 exactly once.
    """
    if world < 1 or not 0 <= rank < world or n_heads < 0:
        raise ValueError("bad rank / world / head count")
    base, extra = divmod(n_heads, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def group_head_range(n_heads: int, group: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, end) range of flattened query heads owned by `rank`
    under grouped-query attention: whole K/V heads, each with its `group`
    query heads, so a K/V head's dK/dV sum stays on one rank and the rank's
    K/V slice is heads [start // group, end // group).
    """
    if group < 1 or n_heads % group != 0:
        raise ValueError("group must divide the query head count")
    a, b = head_range(n_heads // group, rank, world)
    return a * group, b * group


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank scalar (e.g. a timed duration) over all ranks;
    the value itself without an initialised process group."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
