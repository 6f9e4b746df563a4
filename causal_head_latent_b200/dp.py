"""Data-parallel plumbing for the Gated MLA hot path.

Sequences are independent through the whole layer: prefill of one sequence
never reads another's tokens, and decode reads only that sequence's latent
cache ("Gated MLA" page: the per-head attention and the latent cache are per
sequence).  Several GPUs therefore run independent replicas, each on its own
share of the sequences, with no collective on the data path.  This module
holds the host-side pieces: which sequences a rank owns, and the timing
reduction (slowest rank) used by the benchmark.  It works with any
torch.distributed backend (NCCL on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations


def shard_range(n_items: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [begin, end) share of n_items for `rank` of `world`; shares differ
    by at most one item and cover every item exactly once."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n_items, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    """Sum of a per-rank float over the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())
