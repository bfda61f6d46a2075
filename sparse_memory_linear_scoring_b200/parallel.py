"""Multi-GPU plumbing: one process per GPU, (b,h) heads sharded across ranks.

Every (b,h) head of the SDM forward pass has its own slot table, sequence and
gates, and the codebooks are per head, so the heads split across ranks with no
exchange on the data path (the SDM summaries' "Mecanismo Central" item 1: one
table per head).  A rank owns a contiguous range of flat heads f = b*H + h;
the range may start or end inside a batch row, so it is run as at most three
rectangular pieces (a partial row, whole rows, a partial row), each contiguous
in the [B][H] layout and each one sdm_forward call.  This module holds the
host-side pieces: which heads a rank owns and their pieces, the
max-over-ranks reduction used for timing, and assembling per-rank outputs on
every rank.  It works with any torch.distributed backend (NCCL on GPUs, gloo on
CPU).
"""
from __future__ import annotations

from typing import List, NamedTuple, Tuple

import torch
import torch.distributed as dist


def shard_heads(BH_global: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced split of the flat heads: (first flat head, count) of `rank`."""
    if world < 1 or not (0 <= rank < world) or BH_global < 0:
        raise ValueError("bad world/rank")
    base, extra = divmod(BH_global, world)
    f0 = rank * base + min(rank, extra)
    return f0, base + (1 if rank < extra else 0)


class Piece(NamedTuple):
    """Batch rows [b0, b1) x heads [h0, h1): a rectangle of the [B][H] head grid
    whose tensors are contiguous slices (a partial row has b1 = b0 + 1)."""
    b0: int
    b1: int
    h0: int
    h1: int

    @property
    def heads(self) -> int:
        return (self.b1 - self.b0) * (self.h1 - self.h0)


def head_pieces(f0: int, n: int, H: int) -> List[Piece]:
    """The flat heads [f0, f0 + n) of a [B][H] grid as at most three pieces, in
    flat order: the tail of the first row, the whole rows, the head of the last."""
    if H < 1 or f0 < 0 or n < 0:
        raise ValueError("bad head range")
    out: List[Piece] = []
    f, end = f0, f0 + n
    if f < end and f % H:
        b, h = divmod(f, H)
        h1 = min(H, h + (end - f))
        out.append(Piece(b, b + 1, h, h1))
        f += h1 - h
    if end - f >= H:
        nb = (end - f) // H
        out.append(Piece(f // H, f // H + nb, 0, H))
        f += nb * H
    if f < end:
        b = f // H
        out.append(Piece(b, b + 1, 0, end - f))
    return out


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when not distributed)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_heads(t_local: torch.Tensor, BH_global: int) -> torch.Tensor:
    """All ranks' flat-head shards (dim 0, flat head order) concatenated in rank
    order, on every rank: [BH_global, ...].  Shards follow shard_heads; unequal
    shards are padded for the collective."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return t_local
    world = dist.get_world_size()
    sizes = [shard_heads(BH_global, world, r)[1] for r in range(world)]
    m = max(sizes)
    pad = torch.zeros((m,) + tuple(t_local.shape[1:]), dtype=t_local.dtype, device=t_local.device)
    pad[: t_local.shape[0]] = t_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([p[:s] for p, s in zip(parts, sizes)], dim=0)
