"""Pins for oracle.radial: window values, brute force on the tiny grid,
closed-form pair counts, diagonal blocks, dense equality at 64-token blocks."""
import itertools

import numpy as np
import pytest

from oracle import radial
from oracle.pipeline import block_sparse_rows, dense_rows

WAN = dict(w0=1560, w_off=1, full_df=-1)
TINY = dict(w0=64, w_off=0, full_df=1)


@pytest.mark.parametrize("df,expected", [
    # (30*52) / 2^floor(log2(1+df)), evaluated by hand; 1560/16 = 97.5 -> 97
    (0, 1560), (1, 780), (2, 780), (3, 390), (6, 390), (7, 195), (14, 195),
    (15, 97), (20, 97)])
def test_wan_window_values(df, expected):
    assert radial.window(df, 1560, **WAN) == expected


@pytest.mark.parametrize("df,expected", [(0, 64), (1, 64), (2, 32), (3, 32)])
def test_tiny_window_values(df, expected):
    # full attention within |df| <= 1, halved once df has doubled to 2
    assert radial.window(df, 64, **TINY) == expected


def _brute_block_lists(F, H, W, B, params):
    N = F * H * W
    nb = (N + B - 1) // B
    keep = np.zeros((nb, nb), bool)
    for i, j in itertools.product(range(N), range(N)):
        if radial.token_keep(i, j, F, H, W, params):
            keep[i // B, j // B] = True
    return [np.nonzero(keep[b])[0] for b in range(nb)]


@pytest.mark.parametrize("B", [64, 16])
def test_block_lists_equal_brute_force_tiny(B):
    got = radial.block_lists(4, 8, 8, B, TINY)
    ref = _brute_block_lists(4, 8, 8, B, TINY)
    assert len(got) == len(ref)
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)


def test_brute_force_small_wan_like_grid_with_partial_block():
    # 3 frames of 5x6 (S=30) with 16-token blocks: blocks straddle frames and
    # the last block is partial (90 = 5*16 + 10)
    params = dict(w0=30, w_off=1, full_df=-1)
    got = radial.block_lists(3, 5, 6, 16, params)
    ref = _brute_block_lists(3, 5, 6, 16, params)
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)


def test_tiny_b64_keeps_everything():
    lists = radial.block_lists(4, 8, 8, 64, TINY)
    assert all(np.array_equal(l, np.arange(4)) for l in lists)


def test_token_pair_count_closed_form():
    for (F, H, W, params) in [(4, 8, 8, TINY), (21, 30, 52, WAN), (5, 3, 7, dict(w0=21, w_off=1, full_df=0))]:
        S = H * W
        closed = 0
        for fa in range(F):
            for fb in range(F):
                w = min(radial.window(abs(fa - fb), S, **params), S)
                closed += S * S - (S - w) * (S - w + 1)
        assert radial.kept_token_pairs(F, H, W, params) == closed


def test_token_pair_count_brute_tiny():
    F, H, W = 4, 8, 8
    N = F * H * W
    brute = sum(radial.token_keep(i, j, F, H, W, TINY) for i in range(N) for j in range(N))
    assert radial.kept_token_pairs(F, H, W, TINY) == brute


def test_wan_lists_diagonal_and_symmetry():
    lists = radial.block_lists(21, 30, 52, 128, WAN)
    nb = len(lists)
    assert nb == 256
    keep = np.zeros((nb, nb), bool)
    for b, l in enumerate(lists):
        keep[b, l] = True
        assert np.all(np.diff(l) > 0)
    assert keep.diagonal().all()
    assert np.array_equal(keep, keep.T)          # |.| is symmetric
    # O(N log N): far fewer than all pairs, more than the band
    assert 0.3 < keep.mean() < 0.8


def test_tiny_b64_radial_equals_dense():
    rng = np.random.default_rng(0)
    q, k, v = (rng.normal(size=(256, 64)) for _ in range(3))
    lists = radial.block_lists(4, 8, 8, 64, TINY)
    for qb in range(4):
        np.testing.assert_allclose(block_sparse_rows(q, k, v, qb, lists[qb], 64, 64),
                                   dense_rows(q, k, v, qb, 64), rtol=1e-13, atol=1e-14)
