"""Write entropy_calibration.json: alpha/beta of the entropy -> radius map.

The entropy-radius workload asks for a linear entropy -> radius map clamped so
that 9-19% of block pairs are kept ("Token Radius Attention for Efficient
Video Generation": 2. Methodology, The TRA Pipeline, and 4. Experimental
Results for the 9-19% retained interactions).  The map is fixed once from the
oracle's pooled entropies of the seeded inputs: the 5th percentile goes to
radius r_lo, the 95th to the r_hi+1 boundary (oracle.entropy.calibrate).

Calls only oracle/ and synthetic/.  Run:  python tests/golden/make_entropy_calibration.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import entropy  # noqa: E402
from synthetic import make_qkv, workload  # noqa: E402


def main():
    w = workload("tra_entropy")
    e = w["entropy"]
    q, k, _ = make_qkv(w)
    B, d = w["block_q"], w["d"]
    Hs = []
    for h in range(w["heads"]):
        qh = q[h].float().numpy().astype(np.float64)
        kh = k[h].float().numpy().astype(np.float64)
        Hs.append(entropy.pooled_entropy(entropy.block_means(qh, B), entropy.block_means(kh, B),
                                         1.0 / np.sqrt(d)))
    Hs = np.stack(Hs)
    alpha, beta = entropy.calibrate(Hs, e["r_lo"], e["r_hi"])
    cells = entropy.block_cells(w["F"], w["H"], w["W"], B, e["tile_h"], e["tile_w"])
    kept = 0
    near = 0
    for h in range(w["heads"]):
        r = entropy.radius(Hs[h], alpha, beta, e["r_lo"], e["r_hi"])
        kept += sum(len(l) for l in entropy.chebyshev_lists(cells, r))
        near += int(entropy.near_threshold(Hs[h], alpha, beta, e["r_lo"], e["r_hi"]).sum())
    nb = len(cells)
    out = dict(alpha=alpha, beta=beta, r_lo=e["r_lo"], r_hi=e["r_hi"],
               entropy_min=float(Hs.min()), entropy_max=float(Hs.max()),
               block_pair_density=kept / (w["heads"] * nb * nb), near_threshold_rows=near,
               source="oracle.entropy.calibrate on the seeded tra_entropy inputs (seed 0)")
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "entropy_calibration.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
