"""Dual-mode adaptive selection inside a radial prior (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: "DynamicRad: Content-Adaptive Sparse Attention for Long Video
Diffusion" (Abstract): adaptive selection grounded in a radial locality
prior, with two modes, static-ratio (speed first) and dynamic-threshold
(quality first).  The page gives no formulas; readings:
1. Prior: the candidate key blocks of query block b are the static radial
   list of b ("Radial Attention ...", the radial selector of this library,
   oracle/radial.py).
2. Score: pooled attention over the candidates: s_bc = Qbar_b . Kbar_c /
   sqrt(d) with block means over the true token counts, p_bc = softmax over
   the candidates c of b.
3. static-ratio rho: keep the k = ceil(rho * n_cand) candidates of highest
   p (ties to the lower block index); k is taken with a relative slack of
   1e-6 (so that a decimal rho stored in binary does not add one) and kept
   in [1, n_cand].
4. dynamic-threshold theta: sort the candidates by p descending (ties to the
   lower index) and keep the shortest prefix whose cumulative p reaches
   theta (at least one block).
5. The kept ids are listed in ascending order.
Near-threshold rows: a row is reported separately when two candidates whose
order decides membership have p within NEAR relative of each other, or
(dynamic mode) a prefix sum lies within NEAR of theta.

Parity: pinned (tests/test_oracle_dynrad.py): rho = 1 and theta = 1 return
the whole prior; the kept set of static mode has the stated size and holds
the top scores; the dynamic prefix is minimal (its mass reaches theta and
the prefix one shorter does not); both equal brute-force enumeration over
all subsets on tiny inputs; the pooled probabilities sum to 1 and equal
pure-Python loops.
"""
import math

import numpy as np

from . import entropy, radial

NEAR = 1e-5


def candidate_probs(qbar_b, kbar, cands, scale):
    """Softmax over the candidate blocks of the pooled scores (fp64)."""
    s = (kbar[cands] @ qbar_b) * scale
    e = np.exp(s - s.max())
    return e / e.sum()


def order(p, cands):
    """Candidate positions sorted by p descending, ties to the lower block id."""
    return sorted(range(len(cands)), key=lambda i: (-p[i], cands[i]))


def select_row(p, cands, mode, rho=None, theta=None):
    """(kept ids ascending, near flag) for one query block."""
    cands = list(cands)
    n = len(cands)
    if n == 0:
        return [], False
    o = order(p, cands)
    near = False
    if mode == "static":
        k = min(n, max(1, math.ceil(rho * n * (1.0 - 1e-6))))
        if k < n:
            a, b = p[o[k - 1]], p[o[k]]
            near = abs(a - b) <= NEAR * max(a, b)
        kept = [cands[i] for i in o[:k]]
    else:
        acc = 0.0
        kept = []
        for j, i in enumerate(o):
            kept.append(cands[i])
            acc += p[i]
            if abs(acc - theta) <= NEAR:
                near = True
            if acc >= theta:
                break
        if len(kept) < n:
            a, b = p[o[len(kept) - 1]], p[o[len(kept)]]
            near = near or abs(a - b) <= NEAR * max(a, b)
    return sorted(kept), near


def select(q, k, F, H, W, B, radial_params, mode, rho=None, theta=None):
    """Lists of one head: {qb: (ids, near)}."""
    d = q.shape[1]
    qbar = entropy.block_means(q, B)
    kbar = entropy.block_means(k, B)
    prior = radial.block_lists(F, H, W, B, radial_params)
    out = {}
    for b, cands in enumerate(prior):
        p = candidate_probs(qbar[b], kbar, list(cands), 1.0 / math.sqrt(d))
        out[b] = select_row(p, cands, mode, rho, theta)
    return out
