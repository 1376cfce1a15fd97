"""Pins for oracle.attention: dense equality with independent routines,
masked keys contribute nothing, weights behave as the definition says."""
import math

import numpy as np
import pytest
import torch

from oracle import attention
from oracle.pipeline import block_sparse_rows, dense_rows


def _rand(n, m, d, seed=0):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(n, d)), rng.normal(size=(m, d)), rng.normal(size=(m, d))


def _python_loops(q, k, v, scale, w=None):
    out = []
    for i in range(len(q)):
        s = [sum(q[i][c] * k[j][c] for c in range(len(q[i]))) * scale for j in range(len(k))]
        mx = max(s)
        e = [math.exp(x - mx) * (1.0 if w is None else w[j]) for j, x in enumerate(s)]
        den = sum(e)
        out.append([sum(e[j] * v[j][c] for j in range(len(k))) / den for c in range(len(v[0]))])
    return np.array(out)


def test_dense_equals_torch_sdpa_fp64():
    q, k, v = _rand(37, 53, 16)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0]
    got = attention.dense(q, k, v, 1.0 / math.sqrt(16))
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_dense_equals_python_loops():
    q, k, v = _rand(5, 9, 4, seed=1)
    np.testing.assert_allclose(attention.dense(q, k, v, 0.5), _python_loops(q, k, v, 0.5),
                               rtol=1e-12, atol=1e-14)


def test_weighted_equals_python_loops():
    q, k, v = _rand(4, 11, 3, seed=2)
    w = np.random.default_rng(3).uniform(0.5, 7.0, size=11)
    np.testing.assert_allclose(attention.attend(q, k, v, 0.7, w), _python_loops(q, k, v, 0.7, w),
                               rtol=1e-12, atol=1e-14)


def test_constant_weights_are_a_noop():
    q, k, v = _rand(6, 20, 8, seed=4)
    a = attention.attend(q, k, v, 0.3)
    b = attention.attend(q, k, v, 0.3, np.full(20, 9.25))
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


def test_masked_keys_contribute_exactly_zero():
    rng = np.random.default_rng(5)
    N, d, B, U = 96, 8, 32, 16
    q, k, v = (rng.normal(size=(N, d)) for _ in range(3))
    units = [0, 3, 5]                        # tokens 0-15, 48-63, 80-95
    base = block_sparse_rows(q, k, v, 1, units, B, U)
    k2, v2 = k.copy(), v.copy()
    unkept = np.setdiff1d(np.arange(N), np.r_[0:16, 48:64, 80:96])
    k2[unkept] += rng.normal(size=(len(unkept), d)) * 100
    v2[unkept] = rng.normal(size=(len(unkept), d)) * 1e6
    again = block_sparse_rows(q, k2, v2, 1, units, B, U)
    assert np.array_equal(base, again)


def test_full_list_equals_dense_and_partial_tail():
    rng = np.random.default_rng(6)
    N, d, B, U = 70, 8, 32, 16                # ragged: last block 6 tokens
    q, k, v = (rng.normal(size=(N, d)) for _ in range(3))
    units = list(range(5))                   # 5 units of 16 cover 80 > 70 tokens
    for qb in range(3):
        np.testing.assert_allclose(block_sparse_rows(q, k, v, qb, units, B, U),
                                   dense_rows(q, k, v, qb, B), rtol=1e-13, atol=1e-14)


def test_masked_form_matches_gathered_form_and_empty_rows():
    q, k, v = _rand(4, 10, 5, seed=7)
    mask = np.zeros((4, 10), bool)
    mask[0, [1, 4, 7]] = True
    mask[1, :] = True
    mask[2, [9]] = True
    out = attention.attend_masked(q, k, v, 0.4, mask)
    np.testing.assert_allclose(out[0], attention.attend(q[:1], k[[1, 4, 7]], v[[1, 4, 7]], 0.4)[0],
                               rtol=1e-13)
    np.testing.assert_allclose(out[1], attention.attend(q[1:2], k, v, 0.4)[0], rtol=1e-13)
    np.testing.assert_allclose(out[2], v[9], rtol=1e-13)   # single key -> its value
    assert np.array_equal(out[3], np.zeros(5))             # empty key set -> 0
