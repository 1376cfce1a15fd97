"""Difficulty-routed dense/local attention (oracle side).

Source: "Where Compute Matters: Heterogeneous Attention for Efficient Video
Diffusion" (weekinpapers), Abstract: a token-wise difficulty estimate routes
uncertain tokens through dense global attention and the other tokens through
efficient local attention; one parameter sets the trade-off; about 20% of
tokens go through dense attention.

The routed workload replaces the learned uncertainty branch by a seeded
Beta(2,5) score and states a local window of +-1 frame x 16x16 tokens.
Readings:
* one difficulty per token, shared by all heads;
* the routed set R is the ceil(frac * N) tokens of highest difficulty
  (relative slack 1e-6, as for the sampling count), ties broken towards the
  lower token index; compared on the fp32 scores as given;
* a routed query attends to all N keys;
* a local query at (f, h, w) attends to keys (f', h', w') with
  |f' - f| <= win_f, h - win_h <= h' < h + win_h, w - win_w <= w' < w + win_w,
  clipped at the grid edge (16 = 2*8 positions read as half-open; the window
  is not shifted at the edges);
* all tokens are keys on both paths.

Parity: pinned (tests/test_oracle_routed.py): hand-worked tie cases of the
routing rule; window sizes at interior, edge and corner tokens equal the
hand-counted values; the window mask equals a per-pair brute force on a tiny
grid; routed rows equal dense attention.
"""
import math

import numpy as np

from .grid import coords


def route_count(frac, N):
    m = math.ceil(float(frac) * N * (1.0 - 1e-6))
    return max(0, min(N, m))


def route(difficulty, frac):
    """Ascending routed token ids (top ceil(frac*N) by score, ties -> lower id)."""
    dif = np.asarray(difficulty, np.float32)
    N = dif.shape[0]
    k = route_count(frac, N)
    order = np.lexsort((np.arange(N), -dif.astype(np.float64)))
    return np.sort(order[:k]).astype(np.int64)


def window_mask(qtok, ktok, F, H, W, win_f, win_h, win_w):
    """Boolean [len(qtok), len(ktok)]: key inside the query's local window."""
    fq, hq, wq = coords(np.asarray(qtok)[:, None], F, H, W)
    fk, hk, wk = coords(np.asarray(ktok)[None, :], F, H, W)
    return ((np.abs(fk - fq) <= win_f)
            & (hk >= hq - win_h) & (hk < hq + win_h)
            & (wk >= wq - win_w) & (wk < wq + win_w))


def window_keys(t, F, H, W, win_f, win_h, win_w):
    """Key token ids in the local window of token t (ascending)."""
    f, h, w = (int(x) for x in coords(t, F, H, W))
    S = H * W
    out = []
    for ff in range(max(0, f - win_f), min(F, f + win_f + 1)):
        for hh in range(max(0, h - win_h), min(H, h + win_h)):
            base = ff * S + hh * W
            out.extend(range(base + max(0, w - win_w), base + min(W, w + win_w)))
    return np.array(out, dtype=np.int64)
