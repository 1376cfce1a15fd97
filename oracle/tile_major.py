"""Tile-major token layout (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: "Token Radius Attention for Efficient Video Generation" (gist.science
summary), 2. Methodology, The TRA Pipeline, Efficient Execution: the video
tokens are reordered tile by tile so that spatial neighbours (the keys a
query's radius reaches) are contiguous in the sequence, and the token-level
radius masks are then turned into block-sparse masks over that order.

Readings (the page names the layout, not its shape):
1. Tiles are spatial: t_h x t_w tokens of one frame, by default 8 x 16 = 128,
   one block's worth of tokens.
2. Order: frame, then tile row, then tile column, then the row inside the
   tile, then the column inside the tile.  Tiles on the bottom and right
   edges are cut by the grid (ragged, no padding), so the layout is a
   permutation of the N tokens and the sequence length does not change.
3. Blocks are runs of B consecutive positions in the new order, exactly as in
   the raster layout; the last one may be partial.
4. Attention in this layout is attention over the permuted Q, K and V, with
   the output permuted back.  Selectors use each token's (f, h, w) on the
   grid, wherever the token sits in the sequence.

Parity: pinned (tests/test_oracle_tile_major.py): hand-worked orders of a
2 x 4 grid and of a ragged 3 x 3 grid; the layout is a permutation that
keeps every frame contiguous; t_h = 1, t_w = W is the raster order; with
tiles that divide the grid and B = t_h t_w every block is exactly one tile
(closed-form decoding of a position); token-level TRA block lists in this
layout equal a brute-force loop over position pairs; dense and block-sparse
attention commute with the permutation.
"""
import numpy as np

from .grid import coords


def order(F, H, W, th, tw):
    """perm[j] = raster index of the token at tile-major position j."""
    keyed = []
    for t in range(F * H * W):
        f, h, w = (int(x) for x in coords(t, F, H, W))
        keyed.append(((f, h // th, w // tw, h % th, w % tw), t))
    keyed.sort()
    return np.array([t for _, t in keyed], dtype=np.int64)


def position(perm):
    """pos[t] = tile-major position of raster token t (the inverse order)."""
    perm = np.asarray(perm, dtype=np.int64)
    pos = np.empty_like(perm)
    pos[perm] = np.arange(len(perm), dtype=np.int64)
    return pos


def to_layout(x, perm):
    """Rows of x (raster order, tokens on axis 0) in tile-major order."""
    return np.asarray(x)[np.asarray(perm)]


def from_layout(y, perm):
    """Inverse of to_layout: rows in tile-major order back to raster order."""
    y = np.asarray(y)
    out = np.empty_like(y)
    out[np.asarray(perm)] = y
    return out
