"""Token-level entropy -> budget -> radius -> block selector (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: "Token Radius Attention for Efficient Video Generation" (gist.science
summary), 2. Methodology:
* Insight I: a query's retained density follows its attention entropy; the
  token budget is B_i ~ tau * exp(H_i) / N (a fraction of the N keys), so
  query i keeps about n_i = tau * exp(H_i) keys.
* Insight II: the kept keys form a query-centred disk in the spatial domain;
  the radius shrinks with temporal distance delta by phi(delta) =
  exp(-gamma * delta), giving a spatiotemporal support.
* The TRA Pipeline: entropy from a dense warm-up pass, entropy -> budget ->
  base radius -> per-frame 2D disk masks -> token voting into block-sparse
  masks.

Readings (the page prints no formulas beyond the two above):
1. H_i is the natural-log entropy of the dense softmax of query i over all N
   keys with scale 1/sqrt(d).
2. n_i = tau * exp(H_i).
3. The budget is shared among the frames as disks whose radius decays by
   phi: frame f gets n_f = n_i * exp(-2 gamma |f - f_i|) / G(f_i) tokens,
   G(f_i) = sum_{f=0}^{F-1} exp(-2 gamma |f - f_i|), as a disk of squared
   radius r_f^2 = n_f / pi = r0^2 * exp(-2 gamma |f - f_i|) with
   r0^2 = n_i / (pi * G(f_i)) (so sum_f pi r_f^2 = n_i).
4. A frame whose share is below one token (n_f < 1) keeps no key;
   otherwise key j in frame f_j is kept for query i iff
   (h_j - h_i)^2 + (w_j - w_i)^2 <= r_{f_j}^2 (latent grid units).  (Without
   the share rule every frame would keep the key at the query's own (h, w),
   however small its disk: a tube through all frames that alone keeps ~16%
   of the block pairs at the Wan shape, whatever the entropies.)
5. Token voting: key block kb is kept for query block qb iff at least `vote`
   kept (i, j) pairs have i in qb and j in kb.
Near-threshold pairs: |d^2 - r_f^2| <= NEAR * r_f^2 or |n_f - 1| <= NEAR.
A block whose decision depends on such pairs is reported separately
(block_lists returns the ambiguous blocks).  NEAR = 2.5e-5 bounds the
relative distance between an fp32 r_f^2 (or n_f) formed from an entropy
within 2e-5 nats of this one and the fp64 value here:
  * the entropy: |exp(H' - H) - 1| <= 2.0e-5;
  * fp32 arithmetic, u = 2^-24 per rounding, 4u per expf (2 ulp): the
    budget tau * expf(H) 6u (tau rounded to fp32, expf, product); G, a sum
    of F expf terms in frame order, (F + 3)u; pi * G and the division 3u
    (pi rounded, product, quotient); the decay expf and its product 5u; the
    disk test's r_f^2 - dh^2 (dh^2 an exact integer) or the share
    pi * r_f^2 2u: (F + 19)u in all, 2.4e-6 at F = 21 and below 5e-6 for
    F <= 64.
2.0e-5 + 5e-6 = 2.5e-5.

Parity: pinned (tests/test_oracle_tra_token.py): entropy is ln N for equal
logits and ~0 for one dominant logit and equals a pure-Python loop; gamma = 0
gives r0^2 = n / (pi F) and equal per-frame radii; the kept-key count of a
query far from the frame edges equals the Gauss circle count; block lists
equal a brute-force loop over all token pairs on tiny grids; a huge tau keeps
every block, a tiny tau keeps nothing, and a steep decay keeps only the
query's own frame; vote thresholds above the pair count give empty lists;
the near band flags a key at relative distance 1e-5 from the disk edge (or a
share 1e-5 from one token) and not one at 4e-5.
"""
import numpy as np

from .grid import block_range, coords, n_blocks

NEAR = 2.5e-5


def query_entropy(q, k, scale):
    """H_i of softmax_j(scale * q_i . k_j) over all keys, fp64, nats."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    s = (q @ k.T) * scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    p = e / z
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(p > 0, p * np.log(np.where(p > 0, p, 1.0)), 0.0)
    return -t.sum(axis=1)


def frame_weight(fq, F, gamma):
    """G(f_q) = sum over the F frames of exp(-2 gamma |f - f_q|)."""
    f = np.arange(F, dtype=np.float64)
    return float(np.exp(-2.0 * gamma * np.abs(f - fq)).sum())


def radius2(H, fq, F, tau, gamma):
    """Squared disk radius of every frame for a query with entropy H in frame
    fq: array [F]."""
    r0sq = tau * np.exp(H) / (np.pi * frame_weight(fq, F, gamma))
    f = np.arange(F, dtype=np.float64)
    return r0sq * np.exp(-2.0 * gamma * np.abs(f - fq))


def key_keep(i, H_i, F, Hh, W, tau, gamma):
    """(kept, near) boolean masks over all N keys for query i."""
    N = F * Hh * W
    fi, hi, wi = coords(i, F, Hh, W)
    r2 = radius2(H_i, int(fi), F, tau, gamma)
    fj, hj, wj = coords(np.arange(N), F, Hh, W)
    d2 = (hj - hi).astype(np.float64) ** 2 + (wj - wi).astype(np.float64) ** 2
    rf = r2[fj]
    share = np.pi * rf  # n_f: the frame's share of the budget
    kept = (share >= 1.0) & (d2 <= rf)
    near = (np.abs(d2 - rf) <= NEAR * rf) | (np.abs(share - 1.0) <= NEAR)
    return kept, near


def block_lists(H, F, Hh, W, B, tau, gamma, vote=1, qblocks=None, perm=None):
    """Per query block: (ids, ambiguous) where ids are the key blocks kept
    when every pair is decided as stated (ascending) and ambiguous are the
    key blocks whose decision could change if near-threshold pairs went the
    other way.  H: [N] entropies of one head, indexed by raster token.

    perm (optional) is a token layout, perm[j] = raster token at sequence
    position j (oracle/tile_major.py); blocks are then runs of B positions
    of that sequence.  None is the raster layout."""
    N = F * Hh * W
    nb = n_blocks(N, B)
    perm = np.arange(N, dtype=np.int64) if perm is None else np.asarray(perm, dtype=np.int64)
    kb_of = np.empty(N, np.int64)  # block of each raster token
    kb_of[perm] = np.arange(N, dtype=np.int64) // B
    out = {}
    for qb in (range(nb) if qblocks is None else qblocks):
        lo, hi = block_range(qb, B, N)
        cnt = np.zeros(nb, np.int64)
        sure = np.zeros(nb, np.int64)
        maybe = np.zeros(nb, np.int64)
        for i in perm[lo:hi]:
            kept, near = key_keep(i, H[i], F, Hh, W, tau, gamma)
            cnt += np.bincount(kb_of[kept], minlength=nb)
            sure += np.bincount(kb_of[kept & ~near], minlength=nb)
            maybe += np.bincount(kb_of[near], minlength=nb)
        ids = np.nonzero(cnt >= vote)[0]
        # the decision holds whatever the near pairs do iff the sure pairs
        # alone reach the vote, or even all near pairs added do not
        amb = np.nonzero(~((sure >= vote) | (sure + maybe < vote)))[0]
        out[qb] = (ids.astype(np.int64), amb.astype(np.int64))
    return out
