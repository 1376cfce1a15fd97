"""Philox4x32-10 counter-based generator (oracle side, numpy).

Written from Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
1, 2, 3" (SC'11), section on the Philox family: a 4x32-bit counter and a
2x32-bit key; each of 10 rounds multiplies counter words 0 and 2 by two odd
constants, splits each 64-bit product into high and low halves, XORs the high
halves with the other two counter words and the key, and permutes; the key
is bumped by two Weyl constants (golden ratio and sqrt(3)-1, 32-bit) between
rounds.

The pages name no generator; the importance-sampled workload asks for a
counter-based Philox stream per (seed, head, query block).  Use here:

    key     = (seed & 0xffffffff, seed >> 32)
    counter = (j // 4, 0, row, 0),  row = head * n_qb + qblock
    x_j     = output word j % 4
    u_j     = (x_j >> 8) * 2^-24        (exact in fp32 and fp64)

This is the same (seed, subsequence, offset) layout cuRAND documents for
Philox4_32_10 (subsequence in counter words 2-3, element offset in words
0-1).

Parity: pinned (tests/test_oracle_philox.py) against cuRAND's host-side
Philox4_32_10 generator run through its public API, at counters with word 0
and word 2 non-zero and several 64-bit seeds.
"""
import numpy as np

PHILOX_M0 = np.uint64(0xD2511F53)
PHILOX_M1 = np.uint64(0xCD9E8D57)
PHILOX_W0 = np.uint64(0x9E3779B9)
PHILOX_W1 = np.uint64(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)
_SH = np.uint64(32)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10; arguments broadcastable uint32-valued arrays.

    Returns four uint32 arrays.
    """
    c0 = np.asarray(c0, np.uint64) & _MASK
    c1 = np.asarray(c1, np.uint64) & _MASK
    c2 = np.asarray(c2, np.uint64) & _MASK
    c3 = np.asarray(c3, np.uint64) & _MASK
    k0 = np.asarray(k0, np.uint64) & _MASK
    k1 = np.asarray(k1, np.uint64) & _MASK
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + PHILOX_W0) & _MASK
            k1 = (k1 + PHILOX_W1) & _MASK
        p0 = PHILOX_M0 * c0
        p1 = PHILOX_M1 * c2
        c0, c1, c2, c3 = ((p1 >> _SH) ^ c1 ^ k0, p1 & _MASK,
                          (p0 >> _SH) ^ c3 ^ k1, p0 & _MASK)
    return tuple(x.astype(np.uint32) for x in (c0, c1, c2, c3))


def sip_words(seed, row, n):
    """Raw 32-bit words x_j, j = 0..n-1, for one (head, query block) row."""
    seed = int(seed)
    j = np.arange(n, dtype=np.uint64)
    k0 = np.uint64(seed & 0xFFFFFFFF)
    k1 = np.uint64(seed >> 32)
    outs = philox4x32_10(j // np.uint64(4), 0, np.uint64(row), 0, k0, k1)
    stacked = np.stack(outs, axis=0)  # [4, n]
    return stacked[(j % np.uint64(4)).astype(np.int64), np.arange(n)]


def sip_uniforms(seed, row, n):
    """u_j = (x_j >> 8) * 2^-24 in [0, 1), float64 (exact)."""
    x = sip_words(seed, row, n)
    return (x >> np.uint32(8)).astype(np.float64) * (2.0 ** -24)
