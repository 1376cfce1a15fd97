"""Softmax attention restricted to a kept key set, with optional weights (fp64).

Definition.  For query i with kept key set K_i and per-key weights w_k
(1 unless sampled; 1/pi for sampled keys):

    s_ik = q_i . k_k * scale                     (scale = 1/sqrt(d))
    m_i  = max_{k in K_i} s_ik
    O_i  = sum_{k in K_i} w_k exp(s_ik - m_i) v_k / sum_{k in K_i} w_k exp(s_ik - m_i)

Keys outside K_i contribute exactly nothing.  Sources:
* dense softmax self-attention over all tokens: "Token Radius Attention for
  Efficient Video Generation", 1. Problem Statement;
* exact attention on the selected query-key blocks only, pruned blocks
  vanishing from the softmax: same page, 1. Problem Statement (block-level
  methods) and The TRA Pipeline (block-sparse masks); "AB-Attention ..."
  (Glonce), first paragraph;
* reweighting sampled blocks by inverse inclusion probability so that one
  pass estimates dense attention: "AB-Attention ...", method paragraph and
  Why it matters.  The estimate is self-normalised: the same weights enter
  numerator and denominator (reading: the page gives no formula; this is the
  ratio of the two Horvitz-Thompson sums).

scale = 1/sqrt(d) is the standard softmax-attention reading; the pages do
not print it.

An empty key set gives O_i = 0 (reading; the library flags it).

Parity: pinned (tests/test_oracle_attention.py): equals torch's fp64 SDPA and
pure-Python loops when K_i is everything; masked keys are ignored bit for
bit; constant weights are a no-op; weighted form equals pure-Python loops.
"""
import numpy as np


def attend(q, k, v, scale, weights=None):
    """O for queries q [n, d] over one shared key set k, v [m, d]; weights [m]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    if k.shape[0] == 0:
        return np.zeros((q.shape[0], v.shape[1]))
    s = (q @ k.T) * scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    if weights is not None:
        e = e * np.asarray(weights, np.float64)[None, :]
    return (e @ v) / e.sum(axis=1, keepdims=True)


def attend_masked(q, k, v, scale, mask, weights=None):
    """Per-query key sets given as a boolean mask [n, m] over keys k, v."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    out = np.zeros((q.shape[0], v.shape[1]))
    if k.shape[0] == 0:
        return out
    s = (q @ k.T) * scale
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    has = np.isfinite(m[:, 0])
    e = np.where(mask, np.exp(s - np.where(np.isfinite(m), m, 0.0)), 0.0)
    if weights is not None:
        e = e * np.asarray(weights, np.float64)[None, :]
    den = e.sum(axis=1, keepdims=True)
    out[has] = (e[has] @ v) / den[has]
    return out


def dense(q, k, v, scale):
    """Dense attention of every query over every key of one head."""
    return attend(q, k, v, scale)


def flops_kept_pairs(n_pairs, d):
    """Algorithmic FLOPs of attention over n_pairs kept (query, key) pairs:
    2d for q.k plus 2d for p*v, the exponential not counted."""
    return 4.0 * d * n_pairs
