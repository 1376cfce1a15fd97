"""Intra-block clustering selector + inclusion-probability sampling (oracle).

Source: "AB-Attention speeds up video diffusion transformers up to 2.23x, no
training" (Glonce), method paragraph and Key facts: IBCS estimates block
importance by clustering the queries of each query block, without permuting
tokens; SIP samples key/value blocks in proportion to those estimates and
reweights each kept block by its inverse inclusion probability, so that one
pass estimates dense attention; the kernel packs key/value blocks much
smaller than a tile into full tensor-core tiles.

The page prints no formulas.  The importance-sampled workload fixes k = 4,
5 iterations, 128-query blocks, 16-key sub-blocks, ~10% of sub-blocks per
query block, a Philox stream per (seed, head, query block), weights 1/pi.
Readings, in order:

1. Sub-block means Kbar_j over the 16 keys of sub-block j, n_j = true count.
2. k-means per query block (n_b queries): initial centroid c is the query at
   local offset floor(c * n_b / k).  One iteration = assign every query to
   the nearest centroid by squared L2 (tie -> lower centroid index), then
   move each centroid to the mean of its members; an empty cluster keeps its
   centroid.  n_c = member counts of the last assignment.
3. Importance p_j = sum_c (n_c / n_b) * softmax_j(c_c . Kbar_j / sqrt(d)
   + ln n_j): the cluster-weighted share of each centroid's softmax mass
   falling on sub-block j (ln n_j makes a sub-block's pooled logit stand for
   its n_j keys).  sum_j p_j = 1.
4. Target count m = ceil(frac * n_sub) (relative slack 1e-6, so a decimal
   fraction stored in binary does not add one).
5. pi_j = min(1, lambda * p_j) with sum_j pi_j = m (water filling: cap the
   entries with lambda * p_j >= 1, recompute lambda on the rest, repeat).
6. Keep j iff u_j < pi_j, u_j from oracle.philox (independent Poisson
   sampling); each kept sub-block gets weight 1/pi_j on all its keys, stored
   as logw_j = -ln pi_j.

Near-threshold items (|u_j - pi_j| <= 1e-5, or a k-means assignment whose
two smallest distances differ by <= 1e-5 relative) are reported separately.

Parity: pinned (tests/test_oracle_ibcs_sip.py): separable clusters are
recovered; importance sums to 1 and equals pure-Python loops on a tiny case;
water filling meets sum(pi) = m, pi <= 1 and equals a bisection solve;
frac = 1 keeps everything with weight 1 (dense result); the Monte-Carlo mean
over seeds of the Horvitz-Thompson numerator and denominator approaches the
dense values; the k-means margin (relative, floored at a squared distance of
1, minimum over all iterations) equals hand values; near_draws flags exactly
the draws within 1e-5 of pi.
"""
import math

import numpy as np

from .grid import block_range, n_blocks
from .philox import sip_uniforms

NEAR_THRESHOLD = 1e-5


def subblock_means(k, U):
    """Kbar [n_sub, d] fp64 and true counts n_j [n_sub]."""
    k = np.asarray(k, np.float64)
    N = k.shape[0]
    ns = n_blocks(N, U)
    kbar = np.empty((ns, k.shape[1]))
    cnt = np.empty(ns, np.int64)
    for j in range(ns):
        lo, hi = block_range(j, U, N)
        kbar[j] = k[lo:hi].mean(axis=0)
        cnt[j] = hi - lo
    return kbar, cnt


def kmeans(qb, k=4, iters=5):
    """Lloyd's k-means on the queries of one block.

    Returns (centroids [k, d], counts [k], min relative assignment margin).
    """
    qb = np.asarray(qb, np.float64)
    nb = qb.shape[0]
    cent = qb[[(c * nb) // k for c in range(k)]].copy()
    counts = np.zeros(k, np.int64)
    margin = np.inf
    for _ in range(iters):
        d2 = ((qb[:, None, :] - cent[None, :, :]) ** 2).sum(axis=2)  # [nb, k]
        assign = np.argmin(d2, axis=1)  # first minimum -> lower index on ties
        srt = np.sort(d2, axis=1)
        if k > 1:
            rel = (srt[:, 1] - srt[:, 0]) / np.maximum(1.0, srt[:, 0])
            margin = min(margin, float(rel.min()))
        counts = np.bincount(assign, minlength=k)
        for c in range(k):
            if counts[c] > 0:
                cent[c] = qb[assign == c].mean(axis=0)
    return cent, counts, margin


def importance(cent, counts, nb, kbar, n_j, scale):
    """p_j = sum_c (n_c/n_b) softmax_j(c_c . Kbar_j * scale + ln n_j)."""
    s = (np.asarray(cent, np.float64) @ np.asarray(kbar, np.float64).T) * scale
    s = s + np.log(np.asarray(n_j, np.float64))[None, :]
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    sm = e / e.sum(axis=1, keepdims=True)
    wts = np.asarray(counts, np.float64) / float(nb)
    return (wts[:, None] * sm).sum(axis=0)


def target_count(frac, n):
    """m = ceil(frac * n) with a 1e-6 relative slack, clamped to [1, n]."""
    m = math.ceil(float(frac) * n * (1.0 - 1e-6))
    return max(1, min(n, m))


def water_fill(p, m):
    """pi_j = min(1, lambda p_j) with sum pi = m."""
    p = np.asarray(p, np.float64)
    capped = np.zeros(p.shape, bool)
    lam = 0.0
    while True:
        rest = p[~capped].sum()
        if rest <= 0.0:
            break
        lam = (m - capped.sum()) / rest
        new = (~capped) & (lam * p >= 1.0)
        if not new.any():
            break
        capped |= new
    return np.where(capped, 1.0, np.minimum(1.0, lam * p))


def sample(pi, seed, row):
    """Poisson sampling: keep j iff u_j < pi_j.  Returns (kept ids, u)."""
    u = sip_uniforms(seed, row, len(pi))
    return np.nonzero(u < pi)[0].astype(np.int64), u


def near_draws(u, pi):
    """Sub-blocks whose keep decision u_j < pi_j lies within NEAR_THRESHOLD
    of flipping (|u_j - pi_j| <= 1e-5): reported separately, since pi carries
    the rounding of the importance."""
    u = np.asarray(u, np.float64)
    pi = np.asarray(pi, np.float64)
    return np.nonzero(np.abs(u - pi) <= NEAR_THRESHOLD)[0]


def select_row(qb, kbar, n_j, seed, row, k, iters, frac):
    """All steps for one (head, query block).

    Returns dict(ids, logw, pi, u, margin, near_ids).
    """
    d = qb.shape[1]
    scale = 1.0 / np.sqrt(d)
    cent, counts, margin = kmeans(qb, k, iters)
    p = importance(cent, counts, qb.shape[0], kbar, n_j, scale)
    m = target_count(frac, len(p))
    pi = water_fill(p, m)
    ids, u = sample(pi, seed, row)
    near = near_draws(u, pi)
    return dict(ids=ids, logw=-np.log(pi[ids]), pi=pi, u=u, p=p,
                margin=margin, near_ids=near, m=m)


def select(q, k, B, U, seed, head, kiters=5, kk=4, frac=0.10, qblocks=None):
    """Selector for one head over the given query blocks (default: all)."""
    N = q.shape[0]
    nqb = n_blocks(N, B)
    kbar, n_j = subblock_means(k, U)
    rows = {}
    for qbi in (range(nqb) if qblocks is None else qblocks):
        lo, hi = block_range(qbi, B, N)
        rows[qbi] = select_row(np.asarray(q[lo:hi], np.float64), kbar, n_j, seed,
                               head * nqb + qbi, kk, kiters, frac)
    return rows
