"""Write tra_token_calibration.json: the budget constant tau of the token-level
TRA workload.

"Token Radius Attention for Efficient Video Generation" (2. Methodology,
Insight I: a query keeps about tau * exp(H) keys; 4. Experimental Results: TRA
retains 9-19% of attention interactions).  tau is fixed once from the oracle
on the seeded inputs: the per-query entropies of 8 query blocks of head 0
(evenly spaced over the sequence) are computed against all keys, and tau is
bisected (in log space) until those blocks keep 14% of the key blocks on
average.  gamma (temporal decay per frame) and the vote threshold are the
workload's stated readings.

Calls only oracle/ and synthetic/.  Run:  python tests/golden/make_tra_token_calibration.py
"""
import json
import math
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import tra_token  # noqa: E402
from synthetic import make_qkv, workload  # noqa: E402

TARGET = 0.14


def main():
    w = workload("tra_token")
    c = w["tra_token"]
    q, k, _ = make_qkv(w)
    F, H, W, B, d = w["F"], w["H"], w["W"], w["block_q"], w["d"]
    N = F * H * W
    nb = (N + B - 1) // B
    qblocks = [int(x) for x in np.linspace(0, nb - 1, 8).round()]
    qh = q[0].float().numpy().astype(np.float64)
    kh = k[0].float().numpy().astype(np.float64)
    Hq = np.zeros(N)
    for qb in qblocks:
        lo, hi = qb * B, min(N, qb * B + B)
        Hq[lo:hi] = tra_token.query_entropy(qh[lo:hi], kh, 1.0 / math.sqrt(d))

    def density(tau):
        got = tra_token.block_lists(Hq, F, H, W, B, tau, c["gamma"], c["vote"], qblocks)
        return float(np.mean([len(ids) for ids, _ in got.values()])) / nb

    lo, hi = -8.0, 8.0  # log10 tau
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if density(10.0 ** mid) < TARGET:
            lo = mid
        else:
            hi = mid
    tau = float(np.float32(10.0 ** (0.5 * (lo + hi))))
    sel = Hq[np.concatenate([np.arange(qb * B, min(N, qb * B + B)) for qb in qblocks])]
    out = dict(tau=tau, gamma=c["gamma"], vote=c["vote"], target_density=TARGET,
               block_density_sample=density(tau),
               entropy_min=float(sel.min()), entropy_median=float(np.median(sel)),
               entropy_max=float(sel.max()),
               source="oracle.tra_token on 8 query blocks of head 0 of the seeded "
                      "tra_token inputs (seed 0)")
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tra_token_calibration.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
