"""Sharding of the quantize path across ranks (data parallel, no exchange).

The path partitions cleanly: each rank quantizes its own slice and no data
crosses ranks.  Stochastic rounding stays bit-identical to a single-GPU run
because every element draws the Philox word of its global index in the
quantized output view: a rank passes the global index of its slice's first
output element as `elem_offset`.

Slices fall on 32-element boundaries along the split axis, so no block
(32 along a row, 32 down a column, or a 32x32 tile) is cut in two:
  1D-row and 2D layouts split the rows of x[rows, cols]: output rows are
  input rows, the slice's first output element has index row0 * cols;
  the 1D-column layout splits the columns of x: output rows are input
  columns, the slice's first output element has index col0 * rows.
"""
from __future__ import annotations

from dataclasses import dataclass

LAYOUT_1D_ROW, LAYOUT_1D_COL, LAYOUT_2D = 0, 1, 2


@dataclass(frozen=True)
class Shard:
    rank: int
    axis: int          # 0: rows of x are split, 1: columns of x are split
    start: int         # first row (axis 0) or column (axis 1) of x owned by this rank
    size: int          # rows or columns owned
    elem_offset: int   # SR stream index of the slice's first output element


def _split(n_units: int, world: int, rank: int) -> tuple[int, int]:
    base, extra = divmod(n_units, world)
    return rank * base + min(rank, extra), base + (1 if rank < extra else 0)


def shard(rows: int, cols: int, world: int, rank: int, layout: int = LAYOUT_1D_ROW) -> Shard:
    """The slice of x[rows, cols] that `rank` of `world` quantizes."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    if layout == LAYOUT_1D_COL:
        if cols % 32:
            raise ValueError("columns must be a multiple of 32 to shard the 1D-column layout")
        u0, nu = _split(cols // 32, world, rank)
        c0, n = 32 * u0, 32 * nu
        return Shard(rank, 1, c0, n, c0 * rows)
    if rows % 32:
        raise ValueError("rows must be a multiple of 32 to shard on block boundaries")
    u0, nu = _split(rows // 32, world, rank)
    r0, n = 32 * u0, 32 * nu
    return Shard(rank, 0, r0, n, r0 * cols)
