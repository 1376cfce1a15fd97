"""Pins of the tile-major layout oracle ("Token Radius Attention for Efficient
Video Generation", 2. Methodology, The TRA Pipeline, Efficient Execution:
tokens reordered tile by tile so that spatial neighbours are contiguous).

The orders of small grids are worked by hand; the divisible case is checked
against a closed-form decoding of a position into (f, h, w) that does not
use the oracle's sort; block lists are checked against a loop over position
pairs; attention is checked to commute with the permutation."""
import math

import numpy as np
import pytest

from oracle import attention, tile_major, tra_token
from oracle.pipeline import block_sparse_rows, dense_rows


def test_hand_worked_2x4():
    # one frame, rows [0 1 2 3] / [4 5 6 7], 2 x 2 tiles: left tile, then right
    assert tile_major.order(1, 2, 4, 2, 2).tolist() == [0, 1, 4, 5, 2, 3, 6, 7]


def test_hand_worked_ragged_3x3():
    # rows [0 1 2] / [3 4 5] / [6 7 8], 2 x 2 tiles cut by the grid:
    # full tile {0 1 3 4}, right column {2 5}, bottom row {6 7}, corner {8}
    assert tile_major.order(1, 3, 3, 2, 2).tolist() == [0, 1, 3, 4, 2, 5, 6, 7, 8]


def test_two_frames_hand_worked():
    # frame 0 tokens 0..3 then frame 1 tokens 4..7, one 2 x 1 tile column each
    assert tile_major.order(2, 2, 2, 2, 1).tolist() == [0, 2, 1, 3, 4, 6, 5, 7]


@pytest.mark.parametrize("F,H,W,th,tw", [(3, 30, 52, 8, 16), (2, 7, 5, 3, 2), (1, 9, 9, 4, 4)])
def test_permutation_keeps_frames_contiguous(F, H, W, th, tw):
    p = tile_major.order(F, H, W, th, tw)
    N, S = F * H * W, H * W
    assert sorted(p.tolist()) == list(range(N))
    for f in range(F):
        assert set(p[f * S:(f + 1) * S].tolist()) == set(range(f * S, (f + 1) * S))
    pos = tile_major.position(p)
    assert np.array_equal(p[pos], np.arange(N)) and np.array_equal(pos[p], np.arange(N))
    x = np.random.default_rng(0).standard_normal((N, 3))
    assert np.array_equal(tile_major.from_layout(tile_major.to_layout(x, p), p), x)


def test_single_row_tiles_are_raster():
    assert np.array_equal(tile_major.order(3, 5, 7, 1, 7), np.arange(3 * 5 * 7))


def _decode(j, H, W, th, tw):
    """(f, h, w) of tile-major position j when th | H and tw | W."""
    S, T = H * W, th * tw
    f, r = divmod(j, S)
    tile, inner = divmod(r, T)
    tr, tc = divmod(tile, W // tw)
    return f, tr * th + inner // tw, tc * tw + inner % tw


@pytest.mark.parametrize("F,H,W,th,tw", [(2, 16, 32, 8, 16), (3, 6, 8, 2, 4)])
def test_blocks_are_tiles_when_divisible(F, H, W, th, tw):
    p = tile_major.order(F, H, W, th, tw)
    B = th * tw
    for j in range(F * H * W):
        f, h, w = _decode(j, H, W, th, tw)
        assert p[j] == f * H * W + h * W + w
    for b in range(F * H * W // B):
        toks = p[b * B:(b + 1) * B]
        cells = {(t // (H * W), (t % (H * W)) // W // th, (t % W) // tw) for t in toks.tolist()}
        assert len(cells) == 1  # one frame, one tile


def _brute_lists(Hent, F, Hh, W, B, tau, gamma, vote, th, tw):
    """Kept key blocks per query block from a loop over position pairs, with
    positions decoded in closed form (tiles divide the grid)."""
    N = F * Hh * W
    nb = (N + B - 1) // B
    out = {}
    for qb in range(nb):
        cnt = np.zeros(nb, np.int64)
        for i in range(qb * B, min(N, qb * B + B)):
            f, h, w = _decode(i, Hh, W, th, tw)
            ti = f * Hh * W + h * W + w
            kept, _ = tra_token.key_keep(ti, Hent[ti], F, Hh, W, tau, gamma)
            for j in range(N):
                fj, hj, wj = _decode(j, Hh, W, th, tw)
                if kept[fj * Hh * W + hj * W + wj]:
                    cnt[j // B] += 1
        out[qb] = np.nonzero(cnt >= vote)[0].tolist()
    return out


@pytest.mark.parametrize("vote", [1, 3])
def test_token_lists_in_tile_major_match_brute_force(vote):
    F, Hh, W, th, tw = 3, 4, 8, 2, 4
    B = th * tw
    N = F * Hh * W
    Hent = np.random.default_rng(5).uniform(2.0, 3.5, N)
    tau, gamma = 0.6, 0.4
    p = tile_major.order(F, Hh, W, th, tw)
    got = tra_token.block_lists(Hent, F, Hh, W, B, tau, gamma, vote, perm=p)
    ref = _brute_lists(Hent, F, Hh, W, B, tau, gamma, vote, th, tw)
    kept_any = False
    for qb, (ids, _amb) in got.items():
        assert ids.tolist() == ref[qb], qb
        kept_any |= 0 < len(ids) < N // B
    assert kept_any  # neither empty nor dense everywhere


@pytest.mark.parametrize("r2,raster_pairs,tiled_pairs", [(4.5, 46, 100), (100.5, 146, 140)])
def test_block_pair_counts_hand_derived(r2, raster_pairs, tiled_pairs):
    # One 32 x 64 frame, gamma = 0 and G = 1, so every query keeps the disk
    # d^2 <= r2 (tau e^H = pi r2).  B = 128.
    # Raster: block b is rows 2b, 2b+1 (full width).  r = 2.1 reaches rows
    # 2b-2 .. 2b+3, blocks b-1 .. b+1: 2 + 14 * 3 + 2 = 46.  r = 10.02 reaches
    # rows 2b-10 .. 2b+11, blocks b-5 .. b+5: 6+7+8+9+10 + 6*11 + 10+9+8+7+6 = 146.
    # Tiles 8 x 16 (a 4 x 4 tile grid): r = 2.1 reaches the 3 x 3 tile
    # neighbourhood (the diagonal tile at d^2 = 2), clipped: (2+3+3+2)^2 = 100.
    # r = 10.02 reaches tile rows R-2 .. R+2 (the row 9 away) and tile
    # columns C-1 .. C+1 (corner pairs at d^2 = 9^2 + 1 = 82), clipped:
    # (3+4+4+3) * (2+3+3+2) = 140.  The layout that keeps fewer blocks
    # depends on the radius.
    F, Hh, W = 1, 32, 64
    N = F * Hh * W
    Hent = np.full(N, math.log(r2 * math.pi))
    p = tile_major.order(F, Hh, W, 8, 16)
    raster = tra_token.block_lists(Hent, F, Hh, W, 128, 1.0, 0.0)
    tiled = tra_token.block_lists(Hent, F, Hh, W, 128, 1.0, 0.0, perm=p)
    assert sum(len(ids) for ids, _ in raster.values()) == raster_pairs
    assert sum(len(ids) for ids, _ in tiled.values()) == tiled_pairs
    assert not any(len(amb) for _, amb in list(raster.values()) + list(tiled.values()))


def test_attention_commutes_with_the_layout():
    rng = np.random.default_rng(7)
    F, Hh, W, d, B = 2, 6, 8, 16, 16
    N = F * Hh * W
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    p = tile_major.order(F, Hh, W, 2, 4)
    qt, kt, vt = (tile_major.to_layout(x, p) for x in (q, k, v))
    scale = 1.0 / math.sqrt(d)
    # dense: the tile-major output permuted back equals the raster output
    dense_t = np.concatenate([dense_rows(qt, kt, vt, b, B) for b in range(N // B)])
    dense_r = attention.attend(q, k, v, scale)
    assert np.allclose(tile_major.from_layout(dense_t, p), dense_r, rtol=0, atol=1e-12)
    # block-sparse: block b of the tile-major sequence over blocks {b, b+1}
    # equals raster queries over the raster keys those positions hold
    for b in range(N // B - 1):
        got = block_sparse_rows(qt, kt, vt, b, [b, b + 1], B, B)
        keys = p[b * B:(b + 2) * B]
        ref = attention.attend(q[p[b * B:(b + 1) * B]], k[keys], v[keys], scale)
        assert np.allclose(got, ref, rtol=0, atol=1e-12)
