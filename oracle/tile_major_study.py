"""Block-pair share of the token-level lists in raster and tile-major order.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): an fp64 study of the
oracle, not part of the library.

"Token Radius Attention for Efficient Video Generation" (2. Methodology, The
TRA Pipeline, Efficient Execution) reorders tokens tile by tile so that the
keys a query's radius reaches sit in few blocks.  This script measures that
on the seeded token-level workload: for query blocks drawn with a fixed seed
it builds the oracle's lists (tra_token.block_lists) in raster order and in
several tile-major orders (tile_major.order) and prints the share of key
blocks each keeps.  Entropies are the oracle's (query_entropy over all keys
of head 0, with the workload's 12 heads generated).

    python -m oracle.tile_major_study            # 21 x 30 x 52 grid, ~1 min
    python -m oracle.tile_major_study 31 44 80   # wider grid, a few minutes
"""
import math
import sys

import numpy as np

from synthetic import make_qkv, workload

from . import tile_major, tra_token

SHAPES = {(21, 30, 52): [(8, 16), (4, 32), (4, 26), (6, 26), (10, 13), (15, 4), (3, 52)],
          (31, 44, 80): [(8, 16), (4, 32), (11, 10), (4, 40), (2, 80)]}


def study(F, Hh, W, shapes, n_blocks=32, seed=1):
    # all heads are generated: the Q.K scale is fitted over pairs of every head
    w = workload("tra_token", F=F, H=Hh, W=W)
    c = w["tra_token"]
    N, d = w["N"], w["d"]
    q, k, _ = make_qkv(w)
    q0 = q[0].float().numpy().astype(np.float64)
    k0 = k[0].float().numpy().astype(np.float64)
    nqb = (N + 127) // 128
    qbs = sorted(np.random.default_rng(seed).choice(nqb, n_blocks, replace=False).tolist())
    perms = {None: None}
    perms.update({s: tile_major.order(F, Hh, W, *s) for s in shapes})
    need = set()
    for p in perms.values():
        for qb in qbs:
            lo, hi = qb * 128, min(N, qb * 128 + 128)
            need.update(range(lo, hi) if p is None else p[lo:hi].tolist())
    need = np.array(sorted(need))
    H = np.zeros(N)
    for i in range(0, len(need), 256):
        rows = need[i:i + 256]
        H[rows] = tra_token.query_entropy(q0[rows], k0, 1.0 / math.sqrt(d))
    out = {}
    for s, p in perms.items():
        lists = tra_token.block_lists(H, F, Hh, W, 128, c["tau"], c["gamma"], c["vote"],
                                      qblocks=qbs, perm=p)
        out[s] = float(np.mean([len(ids) for ids, _ in lists.values()]) / nqb)
    return out, float(np.median(c["tau"] * np.exp(H[need])))


def main(argv):
    grid = tuple(int(x) for x in argv[:3]) if len(argv) >= 3 else (21, 30, 52)
    n_blocks = 32 if grid == (21, 30, 52) else 24
    shares, budget = study(*grid, SHAPES.get(grid, [(8, 16)]), n_blocks=n_blocks)
    print(f"grid {grid}: {n_blocks} query blocks, median budget {budget:.0f} keys")
    for s, v in shares.items():
        print(f"  {'raster' if s is None else '%dx%d tiles' % s:>12}: {100 * v:.1f}% of block pairs")


if __name__ == "__main__":
    main(sys.argv[1:])
