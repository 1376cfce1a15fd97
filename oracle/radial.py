"""Static radial selector (oracle side).

Source: "Radial Attention to Accelerate Video Generation" (blog), The idea
behind Radial Attention: a static mask drops far-apart token pairs because
their relation decays with distance in space and time; compute falls from
O(N^2) to O(N log N); the same mask is broadcast over batch and heads
(The Build).  The page prints no formula.  Readings:

* Window (token count) at frame distance df:
      w(df) = S                                   if df <= full_df
            = floor(w0 / 2^floor(log2(df + w_off)))  otherwise
  The Wan2.1-1.3B workload states w(df) = (30*52)/2^floor(log2(1+df)):
  w0 = S = 1560, w_off = 1, full_df = -1.  The tiny 4x8x8 workload states
  full attention for |df| <= 1 and halving per doubling: w0 = S = 64,
  w_off = 0, full_df = 1.
* Token pair (i, j) is kept iff |s_i - s_j| < w(|f_i - f_j|), s being the
  flattened spatial index h*W + w inside the frame.  With w = S this keeps
  the whole frame.
* Block pair (qb, kb) is kept iff at least one token pair in it is kept.
  Each block is a union of per-frame runs [a1, a2]; for runs in frames fa,
  fb the closest spatial gap is max(0, b1 - a2, a1 - b2), so the runs share
  a kept pair iff that gap < w(|fa - fb|).

Parity: pinned (tests/test_oracle_radial.py): window values checked against
hand-evaluated values of the two stated formulas; block lists equal brute-
force enumeration of all token pairs on the tiny grid (64- and 16-token
blocks); the token-pair count equals the closed form
sum_{frame pairs} [S^2 - (S - w)(S - w + 1)]; diagonal blocks always kept.
"""
import numpy as np

from .grid import block_frame_intervals, n_blocks


def window(df, S, w0, w_off, full_df):
    """Radial window (in tokens) at non-negative frame distance df."""
    if df <= full_df:
        return S
    n = int(df) + int(w_off)
    if n < 1:
        raise ValueError("radial window undefined: df + w_off < 1 outside the full band")
    e = n.bit_length() - 1  # floor(log2(n)) for integer n >= 1
    return w0 >> e


def token_keep(i, j, F, H, W, params):
    """Token-level radial mask for token indices i, j (scalars)."""
    S = H * W
    fi, si = divmod(int(i), S)
    fj, sj = divmod(int(j), S)
    w = window(abs(fi - fj), S, **params)
    return abs(si - sj) < w


def block_lists(F, H, W, B, params):
    """Kept key-block lists, one per query block (head-independent).

    Returns a list of ascending int arrays.
    """
    N = F * H * W
    S = H * W
    nb = n_blocks(N, B)
    runs = [block_frame_intervals(b, B, N, S) for b in range(nb)]
    lists = []
    for qb in range(nb):
        kept = []
        for kb in range(nb):
            keep = False
            for fa, a1, a2 in runs[qb]:
                for fb, b1, b2 in runs[kb]:
                    gap = max(0, b1 - a2, a1 - b2)
                    if gap < window(abs(fa - fb), S, **params):
                        keep = True
                        break
                if keep:
                    break
            if keep:
                kept.append(kb)
        lists.append(np.array(kept, dtype=np.int64))
    return lists


def kept_token_pairs(F, H, W, params):
    """Number of kept token pairs under the token-level mask (closed form
    per frame pair is not used here: this counts per frame pair by summing
    over spatial offsets)."""
    S = H * W
    total = 0
    for fa in range(F):
        for fb in range(F):
            w = window(abs(fa - fb), S, **params)
            # pairs (a, b) in [0,S)^2 with |a - b| < w: for each offset
            # delta = b - a with |delta| < w there are S - |delta| pairs.
            wmax = min(w, S)
            deltas = np.arange(-(wmax - 1), wmax)
            total += int((S - np.abs(deltas)).sum())
    return total
