"""Data-parallel dw across ranks, bitwise equal to one call over the whole batch.

Two exchanges, both an all-gather in rank order followed by the library's own
pairwise tree (never an all-reduce, whose order depends on the algorithm and
the rank count):

* chunk_split_dw (any split on 256-row boundaries): each rank's backward
  returns its 256-row chunk partials (rmsnorm_bwd_chunks); the ranks' chunk
  partials are gathered in rank order and folded with rn_fold_tree.  dw's
  declared tree is, from its third level up, the pairwise tree over 256-row
  chunks, so this is the one-call dw whenever every rank but the last holds a
  multiple of 256 rows (ranks may hold different counts, or none).
* allgather_fold_dw (equal power-of-two shards): each rank's dw is a perfect
  subtree; only the [width] dw vectors are gathered and folded (rn_fold_rows).


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

from typing import Callable, List, Optional

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


CHUNK_ROWS = 256


def check_chunk_split(rows_local: int, group=None, device=None) -> List[int]:
    """Gathers every rank's row count and checks that the split lies on 256-row
    chunk boundaries: every rank but the last holds a multiple of 256 rows.
    Returns the counts in rank order; raises ValueError on every rank
    otherwise."""
    world = dist.get_world_size(group)
    t = torch.tensor([rows_local], dtype=torch.int64, device=device)
    got = [torch.zeros_like(t) for _ in range(world)]
    dist.all_gather(got, t, group=group)
    rows = [int(g.item()) for g in got]
    if any(r < 0 for r in rows):
        raise ValueError(f"negative row counts {rows}")
    bad = [i for i, r in enumerate(rows[:-1]) if r % CHUNK_ROWS]
    if bad:
        raise ValueError(f"ranks {bad} hold row counts {[rows[i] for i in bad]} that are not "
                         f"multiples of {CHUNK_ROWS}; the exact dw needs a split on {CHUNK_ROWS}-row "
                         "chunk boundaries (only the last rank may hold a ragged count)")
    return rows


def gather_chunk_partials(chunks_local: torch.Tensor, rows_per_rank: List[int],
                          group=None) -> torch.Tensor:
    """All-gathers the ranks' [ceil(rows_r/256), width] chunk partials and
    returns them concatenated in rank order.  Ranks pad their block to the
    largest count for the collective; the padding is dropped again."""
    counts = [-(-r // CHUNK_ROWS) for r in rows_per_rank]
    width = int(chunks_local.shape[1])
    rank = dist.get_rank(group)
    if int(chunks_local.shape[0]) != counts[rank]:
        raise ValueError(f"rank {rank}: {int(chunks_local.shape[0])} chunk partials for "
                         f"{rows_per_rank[rank]} rows, expected {counts[rank]}")
    mx = max(1, max(counts))
    pad = torch.zeros(mx, width, dtype=torch.float32, device=chunks_local.device)
    pad[:counts[rank]] = chunks_local
    outs = [torch.empty_like(pad) for _ in counts]
    dist.all_gather(outs, pad, group=group)
    return torch.cat([o[:c] for o, c in zip(outs, counts)]).contiguous()


def chunk_split_dw(chunks_local: torch.Tensor, rows_local: int, group=None,
                   fold: Optional[Callable[[torch.Tensor], torch.Tensor]] = None,
                   rows_per_rank: Optional[List[int]] = None) -> torch.Tensor:
    """The whole batch's dw from each rank's chunk partials (rank r holds the
    r-th block of rows; see check_chunk_split).  ``fold`` joins the gathered
    rows with the pairwise tree (default: the library's rn_fold_tree).  Pass
    ``rows_per_rank`` from an earlier check_chunk_split to skip the check."""
    if chunks_local.dim() != 2 or chunks_local.dtype != torch.float32:
        raise ValueError("chunks_local must be an fp32 [chunks, width] tensor")
    if rows_per_rank is None:
        rows_per_rank = check_chunk_split(rows_local, group, chunks_local.device)
    gathered = gather_chunk_partials(chunks_local, rows_per_rank, group)
    if gathered.shape[0] == 0:
        raise ValueError("no rows on any rank")
    if fold is None:
        from .ops import rn_fold_tree
        return rn_fold_tree(gathered)
    return fold(gathered)
