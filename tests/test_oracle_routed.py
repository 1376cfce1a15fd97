"""Pins for oracle.routed: tie handling of the routing rule, window sizes at
interior/edge/corner tokens, window mask vs key enumeration."""
import numpy as np
import pytest

from oracle import routed
from oracle.pipeline import routed_rows, dense_rows


def test_route_hand_cases():
    d = np.array([0.5, 0.9, 0.5, 0.1, 0.9], np.float32)
    # top ceil(0.6*5)=3: the two 0.9s, then the lower-index 0.5 (token 0)
    assert list(routed.route(d, 0.6)) == [0, 1, 4]
    # top 2 = both 0.9s
    assert list(routed.route(d, 0.4)) == [1, 4]
    # all equal: lowest indices win
    assert list(routed.route(np.full(6, 0.25, np.float32), 0.5)) == [0, 1, 2]


@pytest.mark.parametrize("frac,N,k", [(0.2, 109120, 21824), (np.float32(0.2), 109120, 21824),
                                      (0.2, 10, 2), (0.0, 10, 0), (1.0, 7, 7)])
def test_route_count(frac, N, k):
    assert routed.route_count(frac, N) == k


@pytest.mark.parametrize("t,size", [
    # grid 31x44x80, window +-1 frame x [h-8, h+8) x [w-8, w+8)
    ((10, 20, 40), 3 * 16 * 16),     # interior
    ((0, 0, 0), 2 * 8 * 8),          # corner: f in {0,1}, h in [0,8), w in [0,8)
    ((30, 43, 79), 2 * 9 * 9),       # far corner: f in {29,30}, h in [35,44), w in [71,80)
    ((15, 3, 40), 3 * 11 * 16),      # near the top edge: h in [0, 11)
])
def test_window_sizes(t, size):
    F, H, W = 31, 44, 80
    tok = t[0] * H * W + t[1] * W + t[2]
    assert len(routed.window_keys(tok, F, H, W, 1, 8, 8)) == size


def test_window_mask_equals_key_enumeration():
    F, H, W = 4, 6, 7
    N = F * H * W
    allk = np.arange(N)
    for t in range(N):
        m = routed.window_mask(np.array([t]), allk, F, H, W, 1, 2, 3)[0]
        assert np.array_equal(np.nonzero(m)[0], routed.window_keys(t, F, H, W, 1, 2, 3))


def test_routed_rows_dense_for_routed_tokens():
    rng = np.random.default_rng(0)
    F, H, W, d = 2, 4, 8, 8
    N = F * H * W
    q, k, v = (rng.normal(size=(N, d)) for _ in range(3))
    flag = np.zeros(N, bool)
    flag[:16] = True
    out = routed_rows(q, k, v, np.arange(16), flag, F, H, W, 1, 2, 2)
    np.testing.assert_allclose(out, dense_rows(q, k, v, 0, 16), rtol=1e-13)
