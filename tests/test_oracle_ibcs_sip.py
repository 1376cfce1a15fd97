"""Pins for oracle.ibcs_sip: k-means on separable clusters, importance as a
distribution and by loops, water filling by bisection, frac=1 gives dense
attention, Horvitz-Thompson unbiasedness over seeds."""
import math

import numpy as np
import pytest

from oracle import ibcs_sip
from oracle.pipeline import block_sparse_rows, dense_rows


def test_kmeans_recovers_separable_clusters():
    rng = np.random.default_rng(0)
    centres = np.array([[10.0, 0, 0], [0, 10.0, 0], [0, 0, 10.0], [-10.0, -10.0, -10.0]])
    sizes = [40, 30, 33, 25]
    pts = np.concatenate([c + 0.1 * rng.normal(size=(n, 3)) for c, n in zip(centres, sizes)])
    perm = rng.permutation(len(pts))
    lab = np.repeat(np.arange(4), sizes)[perm]
    pts = pts[perm]
    cent, counts, margin = ibcs_sip.kmeans(pts, 4, 5)
    # match found clusters to true ones
    for c in range(4):
        true = np.argmin(((centres - cent[c]) ** 2).sum(1))
        assert counts[c] == sizes[true]
        np.testing.assert_allclose(cent[c], pts[lab == true].mean(0), rtol=1e-12)


def test_kmeans_tie_goes_to_lower_index_and_empty_keeps_centroid():
    # identical points: every distance ties, all go to centroid 0; others empty
    pts = np.ones((8, 2))
    cent, counts, _ = ibcs_sip.kmeans(pts, 4, 3)
    assert list(counts) == [8, 0, 0, 0]
    np.testing.assert_array_equal(cent, np.ones((4, 2)))


def test_importance_is_distribution_and_equals_loops():
    rng = np.random.default_rng(1)
    cent = rng.normal(size=(4, 5))
    counts = np.array([3, 0, 10, 3])
    kbar = rng.normal(size=(9, 5))
    n_j = np.array([16] * 8 + [5])
    p = ibcs_sip.importance(cent, counts, 16, kbar, n_j, 0.4)
    assert abs(p.sum() - 1.0) < 1e-13
    ref = np.zeros(9)
    for c in range(4):
        s = [sum(cent[c][t] * kbar[j][t] for t in range(5)) * 0.4 + math.log(n_j[j]) for j in range(9)]
        mx = max(s)
        z = sum(math.exp(x - mx) for x in s)
        for j in range(9):
            ref[j] += counts[c] / 16 * math.exp(s[j] - mx) / z
    np.testing.assert_allclose(p, ref, rtol=1e-12)


def _bisect_pi(p, m):
    lo, hi = 0.0, 1e12
    for _ in range(300):
        mid = 0.5 * (lo + hi)
        if np.minimum(1.0, mid * p).sum() < m:
            lo = mid
        else:
            hi = mid
    return np.minimum(1.0, hi * p)


@pytest.mark.parametrize("m", [1, 5, 20, 40])
def test_water_fill(m):
    rng = np.random.default_rng(2)
    p = rng.dirichlet(np.full(40, 0.3))
    pi = ibcs_sip.water_fill(p, m)
    assert abs(pi.sum() - m) < 1e-9
    assert pi.max() <= 1.0
    np.testing.assert_allclose(pi, _bisect_pi(p, m), atol=1e-9)


@pytest.mark.parametrize("frac,n,m", [(0.10, 7425, 743), (np.float32(0.10), 7425, 743),
                                      (1.0, 7425, 7425), (0.5, 3, 2), (1e-9, 10, 1)])
def test_target_count(frac, n, m):
    # ceil(0.1 * 7425) = ceil(742.5) = 743
    assert ibcs_sip.target_count(frac, n) == m


def test_frac_one_keeps_all_with_unit_weight_and_equals_dense():
    rng = np.random.default_rng(3)
    N, d, B, U = 96, 8, 32, 16
    q, k, v = (rng.normal(size=(N, d)) for _ in range(3))
    rows = ibcs_sip.select(q, k, B, U, seed=11, head=0, frac=1.0)
    for qb, r in rows.items():
        assert list(r["ids"]) == list(range(N // U))
        assert np.all(r["logw"] == 0.0)
        np.testing.assert_allclose(block_sparse_rows(q, k, v, qb, r["ids"], B, U, r["logw"]),
                                   dense_rows(q, k, v, qb, B), rtol=1e-12)


def test_horvitz_thompson_unbiased_over_seeds():
    """Mean over seeds of sum_{kept j} (1/pi_j) A_j equals sum_j A_j, for the
    numerator and denominator of one query's attention (tiny grid, 16 units)."""
    rng = np.random.default_rng(4)
    N, d, U = 256, 16, 16
    q = rng.normal(size=(N, d)) * 1.5
    k = rng.normal(size=(N, d)) * 1.5
    v = rng.normal(size=(N, d))
    qb = q[0:64]
    kbar, n_j = ibcs_sip.subblock_means(k, U)
    cent, counts, _ = ibcs_sip.kmeans(qb, 4, 5)
    p = ibcs_sip.importance(cent, counts, 64, kbar, n_j, 1 / math.sqrt(d))
    pi = ibcs_sip.water_fill(p, 4)
    s = q[0] @ k.T / math.sqrt(d)
    e = np.exp(s - s.max())
    den_units = np.array([e[j * U:(j + 1) * U].sum() for j in range(16)])
    num_units = np.array([e[j * U:(j + 1) * U] @ v[j * U:(j + 1) * U] for j in range(16)])
    n_seeds = 10000
    den_hat = np.zeros(n_seeds)
    num_hat = np.zeros((n_seeds, d))
    for sd in range(n_seeds):
        ids, _ = ibcs_sip.sample(pi, sd, 0)
        den_hat[sd] = (den_units[ids] / pi[ids]).sum()
        num_hat[sd] = (num_units[ids] / pi[ids][:, None]).sum(0)
    # standard error of the mean; 5 sigma
    se = den_hat.std() / math.sqrt(n_seeds)
    assert abs(den_hat.mean() - den_units.sum()) < 5 * se + 1e-12
    se_n = num_hat.std(0) / math.sqrt(n_seeds)
    assert np.all(np.abs(num_hat.mean(0) - num_units.sum(0)) < 5 * se_n + 1e-12)
    # and the expected number kept is m
    kept = np.mean([len(ibcs_sip.sample(pi, sd, 0)[0]) for sd in range(2000)])
    assert abs(kept - 4.0) < 0.15


def test_kmeans_margin_hand_values():
    """The margin is min over queries and iterations of (d2nd - d1st) /
    max(1, d1st), squared L2 distances.  1-D points, k = 2, initial centroids
    q[0] and q[2].

    Points 0, 4, 10, 20 with centroids 0 and 10: the distance pairs are
    (0, 100), (16, 36), (100, 0), (400, 100), so the margins are 100, 20/16,
    100 and 300/100; the minimum is 1.25 (an absolute margin would give 20).
    The second iteration (centroids 2 and 15) gives 29.25, 55.25, 1.56 and
    11.96, so the minimum over both iterations stays 1.25."""
    q = np.array([[0.0], [4.0], [10.0], [20.0]])
    for iters in (1, 2):
        _, _, margin = ibcs_sip.kmeans(q, 2, iters)
        assert abs(margin - 1.25) <= 1e-15, (iters, margin)
    # below a squared distance of 1 the margin is absolute: points 0, 0.3,
    # 0.8, 5 (centroids 0 and 0.8) give pairs (0, .64), (.09, .25), (.64, 0),
    # (25, 17.64): margins .64, .16, .64 and 7.36/17.64; a purely relative
    # margin would give .16/.09 for the second point
    q = np.array([[0.0], [0.3], [0.8], [5.0]])
    _, _, margin = ibcs_sip.kmeans(q, 2, 1)
    assert abs(margin - 0.16) <= 1e-15, margin


def test_kmeans_margin_uses_the_two_nearest_of_four():
    """With k = 4 the margin compares the two smallest of the four distances.
    2-D points; the initial centroids are the points at offsets 0, 1, 2, 3
    (n_b = 4): every point is its own centroid, so the smallest distance is 0
    and each margin is the (floored) distance to its nearest other point."""
    q = np.array([[0.0, 0.0], [3.0, 0.0], [0.0, 10.0], [3.0, 12.0]])
    # nearest-other squared distances: 9, 9, 13, 13 -> margin 9
    _, counts, margin = ibcs_sip.kmeans(q, 4, 1)
    assert list(counts) == [1, 1, 1, 1]
    assert margin == 9.0


def test_near_draws_band():
    pi = np.array([0.3, 0.3, 0.3, 0.3, 0.7, 1.0, 0.05])
    u = np.array([0.3 + 5e-6, 0.3 - 5e-6, 0.3 + 2e-5, 0.3 - 2e-5, 0.7, 0.999995, 0.9])
    assert ibcs_sip.near_draws(u, pi).tolist() == [0, 1, 4, 5]


def test_select_row_reports_its_near_draws():
    rng = np.random.default_rng(5)
    qb = rng.normal(size=(128, 16))
    kbar, n_j = ibcs_sip.subblock_means(rng.normal(size=(512, 16)), 16)
    row = ibcs_sip.select_row(qb, kbar, n_j, 7, 3, 4, 5, 0.25)
    assert row["near_ids"].tolist() == ibcs_sip.near_draws(row["u"], row["pi"]).tolist()
    assert row["ids"].tolist() == np.nonzero(row["u"] < row["pi"])[0].tolist()
