"""Pooled-entropy -> radius -> Chebyshev block selector (oracle side).

Sources: "Token Radius Attention for Efficient Video Generation" (gist.science
summary), 2. Methodology: Insight I (attention entropy measures how diffuse a
query's attention is; a diffuse query needs a larger budget), Insight II (the
budget becomes a radius of a query-centred neighbourhood) and The TRA Pipeline
(entropy -> budget -> radius -> block-sparse mask).

The entropy-radius workload fixes the block form used here: the selector pools
128-query x 128-key blocks, computes the fp32 entropy of the pooled softmax,
maps it linearly to a 3D Chebyshev radius in blocks, and clamps it.  Steps:

1. Pooling: Qbar_b, Kbar_c = means over the block's tokens (true count; the
   last block may be partial).
2. Pooled scores s_bc = Qbar_b . Kbar_c / sqrt(d); p_b = softmax over all key
   blocks c (no size weighting).
3. H_b = -sum_c p_bc ln p_bc, natural log, 0 ln 0 = 0.
4. Radius r_b = clamp(floor(alpha + beta * H_b), r_lo, r_hi).  The workload
   states fp32 entropy, so the decision is taken in fp32: H is rounded to
   fp32 and t = fl32(alpha + fl32(beta * H)) (two separately rounded fp32
   operations), then floor.
5. Block cell (reading: blocks are raster strips, so each is placed at its
   centre token c = b*B + floor((n_b - 1)/2)): (f, floor(h/tile_h),
   floor(w/tile_w)) of token c.  Key block kb is kept for query block qb iff
   max(|df|, |dcell_h|, |dcell_w|) <= r_qb.

Near-threshold rows: |H_b - H*| <= 1e-5 for a threshold H* = (t - alpha)/beta,
t = r_lo+1 .. r_hi, are reported separately (the workload's rule for fp32
entropy close to a radius threshold).

Parity: pinned (tests/test_oracle_entropy.py): entropy is 0 for one-hot and
ln n for uniform p; 0 <= H <= ln n; pooling/scores/entropy equal
pure-Python loops on a tiny grid; a radius covering the grid keeps all
blocks; constant radius gives symmetric lists; lists equal a brute-force
enumeration over cells.
"""
import numpy as np

from .grid import block_range, coords, n_blocks

NEAR_THRESHOLD = 1e-5


def block_means(x, B):
    """Means of x [N, d] over consecutive B-token blocks -> [n_b, d] fp64."""
    x = np.asarray(x, np.float64)
    N = x.shape[0]
    nb = n_blocks(N, B)
    out = np.empty((nb, x.shape[1]))
    for b in range(nb):
        lo, hi = block_range(b, B, N)
        out[b] = x[lo:hi].mean(axis=0)
    return out


def softmax_entropy(p):
    """H = -sum p ln p along the last axis, with 0 ln 0 = 0."""
    p = np.asarray(p, np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(p > 0, p * np.log(np.where(p > 0, p, 1.0)), 0.0)
    return -t.sum(axis=-1)


def pooled_entropy(qbar, kbar, scale):
    """Entropy of softmax_c(Qbar_b . Kbar_c * scale) for every query block."""
    s = (np.asarray(qbar, np.float64) @ np.asarray(kbar, np.float64).T) * scale
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    p = e / e.sum(axis=1, keepdims=True)
    return softmax_entropy(p)


def radius(H, alpha, beta, r_lo, r_hi):
    """Radius per query block; decision in fp32 (see module docstring)."""
    h32 = np.asarray(H, np.float64).astype(np.float32)
    t = np.float32(alpha) + np.float32(beta) * h32   # each op rounded to fp32
    r = np.floor(t).astype(np.int64)
    return np.clip(r, r_lo, r_hi)


def near_threshold(H, alpha, beta, r_lo, r_hi, tol=NEAR_THRESHOLD):
    """True where H lies within tol of a threshold that changes the radius."""
    H = np.asarray(H, np.float64)
    near = np.zeros(H.shape, bool)
    for t in range(r_lo + 1, r_hi + 1):
        hstar = (t - float(np.float32(alpha))) / float(np.float32(beta))
        near |= np.abs(H - hstar) <= tol
    return near


def block_cells(F, H, W, B, tile_h, tile_w):
    """Cell (f, h // tile_h, w // tile_w) of each block's centre token [n_b, 3]."""
    N = F * H * W
    nb = n_blocks(N, B)
    cells = np.empty((nb, 3), np.int64)
    for b in range(nb):
        lo, hi = block_range(b, B, N)
        c = lo + (hi - lo - 1) // 2
        f, h, w = coords(c, F, H, W)
        cells[b] = (f, h // tile_h, w // tile_w)
    return cells


def chebyshev_lists(cells, r):
    """Ascending kept key blocks per query block: D_cheb(qb, kb) <= r[qb]."""
    cells = np.asarray(cells, np.int64)
    out = []
    for qb in range(cells.shape[0]):
        dist = np.abs(cells - cells[qb]).max(axis=1)
        out.append(np.nonzero(dist <= r[qb])[0].astype(np.int64))
    return out


def select(q, k, F, H, W, B, alpha, beta, r_lo, r_hi, tile_h, tile_w):
    """Whole selector for one head: returns (lists, H, r, near)."""
    d = q.shape[1]
    scale = 1.0 / np.sqrt(d)
    Hb = pooled_entropy(block_means(q, B), block_means(k, B), scale)
    r = radius(Hb, alpha, beta, r_lo, r_hi)
    lists = chebyshev_lists(block_cells(F, H, W, B, tile_h, tile_w), r)
    return lists, Hb, r, near_threshold(Hb, alpha, beta, r_lo, r_hi)


def calibrate(entropies, r_lo, r_hi, lo_pct=5.0, hi_pct=95.0):
    """alpha, beta (fp32) that send the lo_pct percentile of the entropies to
    radius r_lo and the hi_pct percentile to the r_hi+1 boundary, so that
    floor() spreads the middle of the distribution over r_lo..r_hi.
    (Reading of "clamped so 9-19% of block pairs are kept": the page gives
    no calibration rule.)"""
    e = np.asarray(entropies, np.float64).ravel()
    h_lo, h_hi = np.percentile(e, lo_pct), np.percentile(e, hi_pct)
    beta = (r_hi + 1 - r_lo) / (h_hi - h_lo)
    alpha = r_lo - beta * h_lo
    return float(np.float32(alpha)), float(np.float32(beta))
