"""Data-parallel plumbing around the step library (host side only).

Each rank trains on its own batch; the mean-loss gradients of the ranks are
averaged (one all-reduce of the contiguous fp32 gradient span) before the
optimizer runs replicated on every rank, so N ranks with B rows each compute
the same update as one rank with N*B rows.  "¿Cómo Entrenar Tu Propio ChatGPT
por $50?" (frequently asked questions) states that single-GPU and 8-GPU runs
give almost identical results; this is the exact form of that equivalence.
"""
from __future__ import annotations


def average_gradients(flat, group=None):
    """In-place mean over ranks of a gradient tensor (SUM then divide: every backend)."""
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return flat
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    flat.div_(dist.get_world_size(group))
    return flat


def max_over_ranks(value: float, device="cpu", group=None) -> float:
    """The slowest rank's value (step times are reported as the max over ranks)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's synthetic batch: distinct per rank, stable across runs."""
    return base + 100 * rank
