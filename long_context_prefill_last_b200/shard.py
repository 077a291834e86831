"""Multi-GPU partitioning of one CRISP layer by KV-head group.

The proxy map, route, selection and sparse attention of a KV group read only
that group's query, key and value heads, so a layer splits across ranks by
KV group with no exchange on the data path: each rank runs the whole path on
its contiguous slice of KV groups (and their query heads) and keeps its slice
of the output, the layout a head-parallel consumer reads. Timing aggregates
as the maximum over ranks.
"""
from __future__ import annotations

from typing import Tuple


def kv_group_range(h_kv: int, world: int, rank: int) -> Tuple[int, int]:
    """[first, last) KV groups of `rank`; groups are dealt in contiguous,
    near-equal slices (the first h_kv % world ranks take one more)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(h_kv, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi


def query_head_range(h_q: int, h_kv: int, world: int, rank: int) -> Tuple[int, int]:
    """[first, last) query heads that belong to the rank's KV groups."""
    g = h_q // h_kv
    lo, hi = kv_group_range(h_kv, world, rank)
    return lo * g, hi * g


def max_over_ranks(value: float, group=None) -> float:
    """Maximum of a per-rank timing over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64)
    if dist.get_backend(group) == "nccl":
        t = t.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
