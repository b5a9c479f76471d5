"""Sequence-split decode over several devices (one process per GPU).

Each rank holds a contiguous slice of every sequence's positions in its
retrieval caches (``DuoKVCache.append_rows``); every rank appends every
token, so the streaming rings are complete everywhere, and one rank (the
last) contributes the streaming heads.  Per layer step each rank decodes its
rows (``decode_rows``), the partial (out, lse) are all-gathered over
``torch.distributed`` (NCCL over NVLink on GPUs), and ``lse_merge`` combines
them exactly.  Host-side arithmetic and plumbing only; the attention and the
merge run in libduo_kv.
"""
from __future__ import annotations

import torch

from .cache import lse_merge


def slice_bounds(capacity_per_rank: int, rank: int) -> tuple[int, int]:
    """Positions [lo, hi) held by `rank`'s retrieval rows when every rank
    reserves `capacity_per_rank` rows: rank r holds r*cap .. (r+1)*cap."""
    lo = rank * capacity_per_rank
    return lo, lo + capacity_per_rank


def local_rows(lengths: torch.Tensor, capacity_per_rank: int, rank: int) -> torch.Tensor:
    """Retrieval rows this rank holds for sequences of the given total lengths
    (int32 [B]): clamp(len - lo, 0, cap)."""
    lo, _ = slice_bounds(capacity_per_rank, rank)
    return (lengths.to(torch.int64) - lo).clamp(0, capacity_per_rank).to(torch.int32)


def gather_partials(out: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather this rank's partial (out [..., d], lse [...]) into
    ([R][..., d], [R][...]) on every rank."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    outs = [torch.empty_like(out) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(outs, out.contiguous(), group=group)
    dist.all_gather(lses, lse.contiguous(), group=group)
    return torch.stack(outs), torch.stack(lses)


def rank_rows(lengths: torch.Tensor, capacity_per_rank: int, rank: int, world: int):
    """What `rank` reads for sequences of the given total lengths (int32
    [B]): its retrieval rows (local_rows) and the streaming ring slots.  Every
    rank holds complete rings, but only the last one reads them, so that each
    streaming key enters the merged result once."""
    rows = local_rows(lengths, capacity_per_rank, rank)
    s_len = lengths if rank == world - 1 else torch.zeros_like(lengths)
    return rows, s_len


def split_decode_step(cache, layer: int, q, lengths, scale: float, capacity_per_rank: int, rank: int,
                      world: int, group=None, gather=None):
    """One decode of one layer for a sequence split over `world` ranks.
    lengths: int32 [B] total tokens held (after the step's append).  Returns
    the merged (out, lse) on every rank.  gather(out, lse, group) collects
    every rank's partials as ([R][...], [R][...]); the default is
    gather_partials over torch.distributed."""
    rows, s_len = rank_rows(lengths, capacity_per_rank, rank, world)
    out, lse = cache.decode_rows(layer, q, rows, scale, s_len=s_len)
    if world == 1:
        return out, lse
    parts_out, parts_lse = (gather or gather_partials)(out, lse, group)
    return lse_merge(parts_out, parts_lse)
