"""Pins of the DynamicRad dual-mode oracle ("DynamicRad: Content-Adaptive
Sparse Attention for Long Video Diffusion", Abstract): selection inside the
radial prior by static ratio or dynamic threshold, against invariants and
brute force over all subsets on tiny inputs."""
import itertools
import math

import numpy as np

from oracle import dynrad, radial


def _probs(n, seed):
    rng = np.random.default_rng(seed)
    p = rng.random(n) + 0.05
    return p / p.sum()


def test_full_ratio_and_full_threshold_keep_the_prior():
    cands = [3, 5, 6, 9, 12]
    p = _probs(5, 0)
    assert dynrad.select_row(p, cands, "static", rho=1.0)[0] == cands
    assert dynrad.select_row(p, cands, "dynamic", theta=1.0)[0] == cands


def test_static_keeps_the_top_scores():
    cands = list(range(10, 30))
    p = _probs(20, 1)
    for rho in (0.1, 0.25, 0.5, 0.9):
        kept, _ = dynrad.select_row(p, cands, "static", rho=rho)
        k = math.ceil(rho * 20 * (1 - 1e-6))
        assert len(kept) == k and kept == sorted(kept)
        pk = sorted(p[[cands.index(c) for c in kept]])
        rest = [p[i] for i, c in enumerate(cands) if c not in kept]
        assert not rest or min(pk) >= max(rest)


def test_dynamic_prefix_is_minimal():
    cands = list(range(15))
    p = _probs(15, 2)
    for theta in (0.2, 0.5, 0.75, 0.95):
        kept, _ = dynrad.select_row(p, cands, "dynamic", theta=theta)
        mass = sum(p[c] for c in kept)
        assert mass >= theta
        # dropping the smallest kept block falls below theta
        smallest = min(kept, key=lambda c: p[c])
        assert mass - p[smallest] < theta


def _brute(p, cands, mode, rho=None, theta=None):
    n = len(cands)
    best = None
    for r in range(1, n + 1):
        for sub in itertools.combinations(range(n), r):
            mass = sum(p[i] for i in sub)
            if mode == "static":
                if r != math.ceil(rho * n * (1 - 1e-6)):
                    continue
                key = (-mass,)
            else:
                if mass < theta:
                    continue
                key = (r, -mass)
            if best is None or key < best[0]:
                best = (key, sub)
        if mode == "dynamic" and best is not None:
            break
    return sorted(cands[i] for i in best[1])


def test_both_modes_equal_brute_force():
    for seed in range(6):
        n = 7
        cands = sorted(np.random.default_rng(seed).choice(40, n, replace=False).tolist())
        p = _probs(n, 10 + seed)
        for rho in (0.3, 0.6):
            got = dynrad.select_row(p, cands, "static", rho=rho)[0]
            assert got == _brute(p, cands, "static", rho=rho)
        for theta in (0.4, 0.8):
            got = dynrad.select_row(p, cands, "dynamic", theta=theta)[0]
            assert got == _brute(p, cands, "dynamic", theta=theta)


def test_pooled_probabilities_equal_loops():
    rng = np.random.default_rng(4)
    qbar = rng.normal(size=8)
    kbar = rng.normal(size=(6, 8))
    cands = [0, 2, 3, 5]
    p = dynrad.candidate_probs(qbar, kbar, cands, 0.5)
    s = [0.5 * sum(qbar[t] * kbar[c, t] for t in range(8)) for c in cands]
    m = max(s)
    e = [math.exp(x - m) for x in s]
    ref = [x / sum(e) for x in e]
    assert np.allclose(p, ref, rtol=1e-13) and abs(p.sum() - 1) < 1e-13


def test_select_stays_inside_the_radial_prior():
    F, H, W, B = 4, 8, 8, 16
    rng = np.random.default_rng(5)
    q = rng.normal(size=(F * H * W, 16))
    k = rng.normal(size=(F * H * W, 16))
    params = dict(w0=64, w_off=0, full_df=1)
    prior = radial.block_lists(F, H, W, B, params)
    for mode, kw in (("static", dict(rho=0.5)), ("dynamic", dict(theta=0.6))):
        got = dynrad.select(q, k, F, H, W, B, params, mode, **kw)
        for b, (ids, _) in got.items():
            assert set(ids) <= set(prior[b]) and len(ids) >= 1


def test_static_near_flag_on_close_scores():
    """Static ratio keeps 2 of 4; the kept-last and dropped-first candidates
    are near when their probabilities differ by <= 1e-5 relative."""
    cands = [10, 11, 12, 13]
    for rel, near in ((0.5e-5, True), (2e-5, False)):
        p = np.array([0.4, 0.3, 0.3 * (1 - rel), 0.1])
        kept, flag = dynrad.select_row(p, cands, "static", rho=0.5)
        assert kept == [10, 11] and bool(flag) == near, (rel, flag)


def test_dynamic_near_flag_on_prefix_mass_and_close_scores():
    cands = [3, 5, 8, 9]
    # prefix mass 0.700004 reaches theta = 0.7 within 1e-5: near
    kept, flag = dynrad.select_row(np.array([0.4, 0.3 + 4e-6, 0.2, 0.1]), cands, "dynamic",
                                   theta=0.7)
    assert kept == [3, 5] and flag
    # 0.70003 is 3e-5 past theta, and the next candidate is far: not near
    kept, flag = dynrad.select_row(np.array([0.4, 0.3 + 3e-5, 0.2, 0.1]), cands, "dynamic",
                                   theta=0.7)
    assert kept == [3, 5] and not flag
    # a prefix 5e-6 short of theta is near too (one more rounding step and it
    # would have stopped there)
    kept, flag = dynrad.select_row(np.array([0.4, 0.3 - 5e-6, 0.2, 0.1]), cands, "dynamic",
                                   theta=0.7)
    assert kept == [3, 5, 8] and flag
    # the last kept and the first dropped candidate within 1e-5 relative
    for rel, near in ((0.5e-5, True), (2e-5, False)):
        p = np.array([0.5, 0.3, 0.3 * (1 - rel), 0.05])
        kept, flag = dynrad.select_row(p, cands, "dynamic", theta=0.75)
        assert kept == [3, 5] and bool(flag) == near, (rel, flag)
