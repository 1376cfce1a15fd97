"""Whole-path oracle per workload: selector lists, then attention rows.

Each function takes one head's q, k, v (any float array type; widened to
fp64) and returns fp64 outputs for the requested query blocks, so that tests
can check sampled blocks of full-size workloads and whole small ones.
"""
import numpy as np

from . import attention, entropy, ibcs_sip, radial, routed
from .grid import block_range, n_blocks, unit_tokens


def as64(x):
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, np.float64)


def block_sparse_rows(q, k, v, qb, units, B, U, logw=None, scale=None):
    """O for query block qb attending to the tokens of the given KV units.

    logw (optional) holds -ln(pi) per unit: every key of the unit gets
    weight exp(logw) = 1/pi.
    """
    q, k, v = as64(q), as64(k), as64(v)
    N, d = q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    lo, hi = block_range(qb, B, N)
    toks = unit_tokens(units, U, N)
    wts = None
    if logw is not None:
        per_unit = [np.full(min((u + 1) * U, N) - u * U, np.exp(lw))
                    for u, lw in zip(units, logw)]
        wts = np.concatenate(per_unit) if per_unit else np.zeros(0)
    return attention.attend(q[lo:hi], k[toks], v[toks], scale, wts)


def dense_rows(q, k, v, qb, B, scale=None):
    q, k, v = as64(q), as64(k), as64(v)
    N, d = q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    lo, hi = block_range(qb, B, N)
    return attention.attend(q[lo:hi], k, v, scale)


def routed_rows(q, k, v, toks, routed_flag, F, H, W, win_f, win_h, win_w, scale=None):
    """O for the given query tokens under routing (flag[t] True -> dense)."""
    q, k, v = as64(q), as64(k), as64(v)
    N, d = q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.zeros((len(toks), d))
    for r, t in enumerate(toks):
        if routed_flag[t]:
            out[r] = attention.attend(q[t:t + 1], k, v, scale)[0]
        else:
            keys = routed.window_keys(t, F, H, W, win_f, win_h, win_w)
            out[r] = attention.attend(q[t:t + 1], k[keys], v[keys], scale)[0]
    return out


def kept_pairs_block_lists(lists, B, U, N, heads=1):
    """Algorithmic kept (query, key) pairs of block/unit lists, true lengths."""
    nqb = n_blocks(N, B)
    total = 0
    for qb in range(nqb):
        lo, hi = block_range(qb, B, N)
        keys = sum(min((u + 1) * U, N) - u * U for u in lists[qb])
        total += (hi - lo) * keys
    return total * heads


__all__ = ["block_sparse_rows", "dense_rows", "routed_rows", "kept_pairs_block_lists",
           "radial", "entropy", "ibcs_sip", "routed", "attention"]
