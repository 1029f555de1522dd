"""Model of the declared dw reduction tree, in IEEE fp32 on the CPU.

The norm contract (RL-Kernel RFC #415, section 4 "Numerical contract": a declared
fp32 accumulator, an addition order that does not depend on batch size,
position, packing, launch geometry or SM count, and no split reductions unless
the merge tree is itself fixed) leaves the tree's shape to the implementation.
The library declares this one:

  1. leaf = 32 consecutive rows, leaf l = rows [32 l, 32 l + 32) of the call;
     its partial is the ascending left fold of the rows' fp32 contributions,
     started from the first row (not from 0);
  2. the leaf partials are combined by a level-by-level pairwise tree: at
     each level node 2i is added to node 2i+1 (left + right) and an odd last
     node is carried up unchanged; missing nodes are absent, never +0.

Its shape depends on the row count only.  Nodes grouped in aligned blocks of a
power of two form perfect subtrees (the first levels of the tree pair only
inside such blocks), which is what lets the GPU fold 256-row chunks -- or any
other aligned power-of-two block -- in any order and still give these bits.

A row's contribution is what the backward returns as dw when called on that row
alone (a one-row leaf needs no addition), so the batch dw must equal this model
applied to the one-row dws bitwise.  numpy float32 adds are IEEE
round-to-nearest-even with no fused multiply-add.
"""
from __future__ import annotations

from typing import Callable, List, Sequence

import numpy as np

LEAF_ROWS = 32


def left_fold(items: Sequence, add: Callable):
    acc = items[0]
    for v in items[1:]:
        acc = add(acc, v)
    return acc


def pairwise_tree(nodes: Sequence, add: Callable):
    nodes = list(nodes)
    assert nodes, "empty tree"
    while len(nodes) > 1:
        nxt = [add(nodes[i], nodes[i + 1]) for i in range(0, len(nodes) - 1, 2)]
        if len(nodes) % 2:
            nxt.append(nodes[-1])
        nodes = nxt
    return nodes[0]


def _f32_add(a, b):
    return (np.asarray(a, dtype=np.float32) + np.asarray(b, dtype=np.float32)).astype(np.float32)


def dw_tree(contribs: np.ndarray, add: Callable = _f32_add) -> np.ndarray:
    """contribs: [rows, width] fp32 one-row dws -> the declared batch dw."""
    contribs = np.asarray(contribs, dtype=np.float32)
    rows = contribs.shape[0]
    leaves: List = [left_fold([contribs[r] for r in range(s, min(rows, s + LEAF_ROWS))], add)
                    for s in range(0, rows, LEAF_ROWS)]
    return np.asarray(pairwise_tree(leaves, add), dtype=np.float32)


def tree_shape(n: int) -> str:
    """The tree over n nodes written out, e.g. tree_shape(5) == '(((0+1)+(2+3))+4)'."""
    return pairwise_tree([str(i) for i in range(n)], lambda a, b: f"({a}+{b})")


CHUNK_ROWS = 256


def chunk_partials(contribs: np.ndarray, add: Callable = _f32_add) -> np.ndarray:
    """contribs: [rows, width] fp32 one-row dws -> the 256-row chunk partials
    [ceil(rows/256), width]: chunk c is the declared tree over the leaves of
    rows [256 c, 256 c + 256) (fewer in a ragged last chunk)."""
    contribs = np.asarray(contribs, dtype=np.float32)
    return np.stack([dw_tree(contribs[s:s + CHUNK_ROWS], add)
                     for s in range(0, contribs.shape[0], CHUNK_ROWS)])
