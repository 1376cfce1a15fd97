"""Fit the cubic used for 2^f, f in [-1/2, 1/2], by the Remez exchange
algorithm on relative error (E. Remez, 1934; see e.g. Cheney, "Introduction
to Approximation Theory", ch. 3).  The kernel writes x = j + f with j the
nearest integer and evaluates 2^x = p(f) * 2^j, adding j to the exponent
bits.  Prints the coefficients (c0..c3) and the maximum relative error of
the exact polynomial and of its fp32 Horner evaluation.

    python sparse_spatiotemporal_attention_video_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def remez(n, lo, hi, iters=40):
    m = n + 2
    x = (lo + hi) / 2 - (hi - lo) / 2 * np.cos(np.pi * np.arange(m) / (m - 1))
    c = None
    for _ in range(iters):
        A = np.zeros((m, m))
        for i in range(m):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2 ** x[i]
        c = np.linalg.solve(A, 2 ** x)[:n + 1]
        g = np.linspace(lo, hi, 400001)
        err = (np.polyval(c[::-1], g) - 2 ** g) / 2 ** g
        ext = [0] + [i for i in range(1, len(g) - 1)
                     if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) < 0] + [len(g) - 1]
        if len(ext) != m:
            break
        x = g[ext]
    return c


if __name__ == "__main__":
    c = remez(3, -0.5, 0.5)
    c32 = [np.float32(v) for v in c]
    g = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.float32(c32[3])
    for cc in c32[2::-1]:
        p = (p * g + cc).astype(np.float32)
    print("coefficients:", ", ".join(f"{float(v):.9g}f" for v in c32))
    print("max rel error (fp32 Horner):",
          float(np.abs(p.astype(np.float64) / 2.0 ** g.astype(np.float64) - 1).max()))
