"""Data-parallel dw across ranks, bitwise equal to one call over the whole batch.

Rows are independent, so y, rstd, dx and dz need no communication when a batch
is split across ranks.  dw is a sum over rows; its declared reduction is a
pairwise tree over 32-row leaves, and a reduction whose order depended on the
rank count (an all-reduce) would break the contract that the order depends on
the row count only (RL-Kernel RFC #415, section 4 "Numerical contract", points
2 and 3).

When every rank holds the same power-of-two number of leaves and the ranks'
blocks are in batch order, each rank's dw (the root of the tree over its own
leaves) is a perfect subtree of the tree over all leaves, and the tree's
remaining levels are the pairwise tree over the ranks' dw in rank order.  So:
all-gather the [width] dw vectors (not an all-reduce), then fold them with the
same tree (rn_fold_rows).  Every rank computes the identical result.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

LEAF_ROWS = 32


def _is_pow2(v: int) -> bool:
    return v > 0 and (v & (v - 1)) == 0


def check_shard_rows(rows_local: int, group=None, device=None) -> int:
    """All ranks' row counts must be equal, a multiple of 32, with a power-of-two
    number of leaves.  Returns the number of ranks; raises ValueError otherwise."""
    world = dist.get_world_size(group)
    t = torch.tensor([rows_local], dtype=torch.int64, device=device)
    got = [torch.zeros_like(t) for _ in range(world)]
    dist.all_gather(got, t, group=group)
    rows = [int(g.item()) for g in got]
    if len(set(rows)) != 1:
        raise ValueError(f"ranks hold different row counts {rows}; the exact dw fold needs equal shards")
    r = rows[0]
    if r % LEAF_ROWS or not _is_pow2(r // LEAF_ROWS):
        raise ValueError(f"{r} rows per rank is not a power-of-two number of {LEAF_ROWS}-row leaves")
    return world


def fold_gathered_dw(dw_local: torch.Tensor, group=None,
                     fold: Optional[Callable[[torch.Tensor], torch.Tensor]] = None
                     ) -> torch.Tensor:
    """All-gathers the ranks' [width] dw in rank order and joins them with the
    pairwise tree (``fold``; default: the library's rn_fold_rows).  The caller
    vouches for the shard shapes (see check_shard_rows)."""
    world = dist.get_world_size(group)
    if world > 256:
        raise ValueError("at most 256 ranks")
    outs = [torch.empty_like(dw_local) for _ in range(world)]
    dist.all_gather(outs, dw_local.contiguous(), group=group)
    gathered = torch.stack(outs)           # [world, width], rank order
    if fold is None:
        from .ops import rn_fold_rows
        return rn_fold_rows(gathered)
    return fold(gathered)


def allgather_fold_dw(dw_local: torch.Tensor, rows_local: int, group=None,
                      fold: Optional[Callable[[torch.Tensor], torch.Tensor]] = None
                      ) -> torch.Tensor:
    """The dw of the whole batch from each rank's dw (rank r holds the r-th block
    of rows), after checking the shard shapes on every rank."""
    if dw_local.dim() != 1 or dw_local.dtype != torch.float32:
        raise ValueError("dw_local must be an fp32 [width] tensor")
    check_shard_rows(rows_local, group, dw_local.device)
    return fold_gathered_dw(dw_local, group, fold)
