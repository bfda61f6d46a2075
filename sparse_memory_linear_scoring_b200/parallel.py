"""Multi-GPU plumbing: one process per GPU, heads sharded across ranks.

Every (b,h) head of the SDM forward pass has its own slot table, sequence and
gates, and the codebooks are per head, so a batch splits across ranks with no
exchange on the data path.  This module holds the host-side pieces: which batch
rows a rank owns, the max-over-ranks reduction used for timing, and assembling
per-rank outputs on every rank.  It works with any torch.distributed backend
(NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

from typing import Tuple

import torch
import torch.distributed as dist


def shard_batch(B_global: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced split of batch rows: (first row, row count) of `rank`."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("bad world/rank")
    base, extra = divmod(B_global, world)
    b0 = rank * base + min(rank, extra)
    return b0, base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when not distributed)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_batch(t_local: torch.Tensor, B_global: int) -> torch.Tensor:
    """All ranks' batch shards (dim 0) concatenated in rank order, on every rank.
    Shards follow shard_batch; unequal shards are padded for the collective."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return t_local
    world = dist.get_world_size()
    sizes = [shard_batch(B_global, world, r)[1] for r in range(world)]
    m = max(sizes)
    pad = torch.zeros((m,) + tuple(t_local.shape[1:]), dtype=t_local.dtype, device=t_local.device)
    pad[: t_local.shape[0]] = t_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([p[:s] for p, s in zip(parts, sizes)], dim=0)
