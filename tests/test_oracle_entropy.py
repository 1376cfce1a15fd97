"""Pins for oracle.entropy: entropy closed forms, brute force of pooling and
scores on a tiny grid, Chebyshev lists by enumeration, radius edge cases."""
import math

import numpy as np
import pytest

from oracle import entropy
from oracle.grid import coords


def test_entropy_one_hot_is_zero():
    p = np.zeros(17)
    p[5] = 1.0
    assert entropy.softmax_entropy(p) == 0.0


@pytest.mark.parametrize("n", [1, 2, 7, 256])
def test_entropy_uniform_is_log_n(n):
    assert abs(entropy.softmax_entropy(np.full(n, 1.0 / n)) - math.log(n)) < 1e-13


def test_entropy_two_point_hand_value():
    # p = (1/4, 3/4): H = -(0.25 ln 0.25 + 0.75 ln 0.75) = 0.5623351446188083
    assert abs(entropy.softmax_entropy(np.array([0.25, 0.75])) - 0.5623351446188083) < 1e-15


def test_pooled_entropy_bounds():
    rng = np.random.default_rng(0)
    H = entropy.pooled_entropy(rng.normal(size=(9, 8)) * 3, rng.normal(size=(13, 8)) * 3, 0.35)
    assert np.all(H >= 0) and np.all(H <= math.log(13) + 1e-12)


def _loops(q, k, F, Hh, W, B):
    N, d = q.shape
    nb = (N + B - 1) // B
    def mean(x, b):
        toks = [t for t in range(b * B, min((b + 1) * B, N))]
        return [sum(x[t][c] for t in toks) / len(toks) for c in range(d)]
    qbar = [mean(q, b) for b in range(nb)]
    kbar = [mean(k, b) for b in range(nb)]
    out = []
    for b in range(nb):
        s = [sum(qbar[b][c] * kbar[c2][c] for c in range(d)) / math.sqrt(d) for c2 in range(nb)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        z = sum(e)
        out.append(-sum((x / z) * math.log(x / z) for x in e if x > 0))
    return np.array(out)


def test_pooled_entropy_equals_loops_tiny_ragged():
    rng = np.random.default_rng(1)
    F, H, W, B, d = 3, 4, 5, 16, 6          # N = 60, last block 12 tokens
    q = rng.normal(size=(60, d)) * 2
    k = rng.normal(size=(60, d)) * 2
    got = entropy.pooled_entropy(entropy.block_means(q, B), entropy.block_means(k, B), 1 / math.sqrt(d))
    np.testing.assert_allclose(got, _loops(q, k, F, H, W, B), rtol=1e-12)


def test_radius_decision_hand_values():
    # alpha=-1, beta=2: H=1.2 -> 1.4 -> 1; H=2.6 -> 4.2 -> 4 -> clamp 3; H=0.1 -> -0.8 -> -1 -> clamp 0
    r = entropy.radius(np.array([1.2, 2.6, 0.1]), -1.0, 2.0, 0, 3)
    assert list(r) == [1, 3, 0]


def test_cells_hand_values():
    # 2 frames of 4x8 (S=32), B=16: block 0 = tokens 0..15, centre 7 = (0,0,7)
    # -> cell (0, 0, 7//4=1) with tile (2, 4); block 3 = tokens 48..63,
    # centre 55 = (1, 2, 7) -> (1, 1, 1)
    cells = entropy.block_cells(2, 4, 8, 16, 2, 4)
    assert tuple(cells[0]) == (0, 0, 1)
    assert tuple(cells[3]) == (1, 1, 1)


def test_chebyshev_lists_brute_force():
    F, H, W, B, th, tw = 5, 6, 10, 16, 2, 4
    cells = entropy.block_cells(F, H, W, B, th, tw)
    rng = np.random.default_rng(2)
    r = rng.integers(0, 3, size=len(cells))
    got = entropy.chebyshev_lists(cells, r)
    N = F * H * W
    for qb in range(len(cells)):
        ref = []
        cq = coords(qb * B + (min(B, N - qb * B) - 1) // 2, F, H, W)
        for kb in range(len(cells)):
            ck = coords(kb * B + (min(B, N - kb * B) - 1) // 2, F, H, W)
            dist = max(abs(int(cq[0]) - int(ck[0])), abs(int(cq[1]) // th - int(ck[1]) // th),
                       abs(int(cq[2]) // tw - int(ck[2]) // tw))
            if dist <= r[qb]:
                ref.append(kb)
        assert list(got[qb]) == ref


def test_radius_covering_grid_keeps_all_and_constant_radius_symmetric():
    F, H, W, B = 21, 30, 52, 128
    cells = entropy.block_cells(F, H, W, B, 8, 16)
    full = entropy.chebyshev_lists(cells, np.full(len(cells), F + 10))
    assert all(len(l) == len(cells) for l in full)
    two = entropy.chebyshev_lists(cells, np.full(len(cells), 2))
    keep = np.zeros((len(cells),) * 2, bool)
    for b, l in enumerate(two):
        keep[b, l] = True
    assert np.array_equal(keep, keep.T) and keep.diagonal().all()


def test_near_threshold_flags():
    alpha, beta = -1.0, 2.0           # thresholds at H* = 1.0 (t=1) and 1.5 (t=2)
    H = np.array([1.0 + 5e-6, 1.5 - 2e-6, 1.2, 1.0 + 2e-5])
    assert list(entropy.near_threshold(H, alpha, beta, 0, 2)) == [True, True, False, False]


def test_calibrate_hand_worked():
    """Entropies 0..9 (any order): with linear interpolation between order
    statistics the 5th percentile is 0.45 and the 95th is 8.55.  Mapping them
    to radius 1 and to the boundary of radius 3 (r_hi + 1 with r_hi = 2)
    gives beta = 2 / 8.1 = 20/81 and alpha = 1 - 0.45 * 20/81 = 8/9, each
    rounded to fp32."""
    e = np.array([7.0, 2.0, 9.0, 0.0, 4.0, 1.0, 8.0, 3.0, 6.0, 5.0])
    alpha, beta = entropy.calibrate(e, 1, 2)
    assert alpha == float(np.float32(8.0 / 9.0))
    assert beta == float(np.float32(20.0 / 81.0))


def test_calibrate_maps_percentiles_to_the_radius_range():
    rng = np.random.default_rng(4)
    e = 5.4 + 0.1 * rng.random(3000)
    for r_lo, r_hi in ((1, 2), (0, 3), (2, 6)):
        alpha, beta = entropy.calibrate(e, r_lo, r_hi)
        h5, h95 = np.percentile(e, 5), np.percentile(e, 95)
        assert abs(alpha + beta * h5 - r_lo) <= 1e-5 * (1 + abs(alpha))
        assert abs(alpha + beta * h95 - (r_hi + 1)) <= 1e-5 * (1 + abs(alpha))
        r = entropy.radius(e, alpha, beta, r_lo, r_hi)
        # the lowest 5% sit at r_lo, the top 5% are clamped at r_hi, and the
        # middle spreads over every radius in between
        assert set(np.unique(r).tolist()) == set(range(r_lo, r_hi + 1))
        assert (r[e < h5 - 1e-6] == r_lo).all()
        assert (r[e > h95 + 1e-6] == r_hi).all()
