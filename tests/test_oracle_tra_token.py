"""Pins of the token-level entropy -> radius -> block selector oracle
("Token Radius Attention for Efficient Video Generation", 2. Methodology:
Insight I, Insight II, The TRA Pipeline), against closed forms, invariants
and brute force on tiny grids."""
import math

import numpy as np
import pytest

from oracle import tile_major, tra_token


def test_entropy_of_equal_logits_is_ln_n():
    rng = np.random.default_rng(0)
    q = rng.normal(size=(5, 8))
    k = np.tile(rng.normal(size=(1, 8)), (37, 1))  # every key identical
    H = tra_token.query_entropy(q, k, 0.3)
    assert np.allclose(H, math.log(37), atol=1e-12)


def test_entropy_of_one_dominant_logit_is_near_zero():
    q = np.zeros((1, 4))
    q[0, 0] = 1.0
    k = np.zeros((50, 4))
    k[7, 0] = 200.0  # logit 200 against 0 for the 49 others
    H = tra_token.query_entropy(q, k, 1.0)
    # exact value: p = 1/(1 + 49 e^-200); H ~ 49 * 200 * e^-200
    assert 0.0 <= H[0] < 1e-80


def test_entropy_equals_loops():
    rng = np.random.default_rng(1)
    q = rng.normal(size=(3, 6))
    k = rng.normal(size=(11, 6))
    s = 0.7
    H = tra_token.query_entropy(q, k, s)
    for i in range(3):
        logits = [s * sum(q[i, t] * k[j, t] for t in range(6)) for j in range(11)]
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        z = sum(w)
        ref = -sum((x / z) * math.log(x / z) for x in w)
        assert abs(H[i] - ref) < 1e-12


def test_radius_without_decay_is_uniform():
    F, tau, H = 7, 3.0, 2.5
    r2 = tra_token.radius2(H, 2, F, tau, 0.0)
    r0sq = tau * math.exp(H) / (math.pi * F)
    assert np.allclose(r2, r0sq, rtol=1e-14)
    # the disks of all frames hold n = tau e^H tokens in the continuous sense
    assert abs(math.pi * r2.sum() - tau * math.exp(H)) < 1e-9


def test_radius_decay_by_frame_distance():
    F, gamma = 9, 0.4
    r2 = tra_token.radius2(1.0, 4, F, 2.0, gamma)
    for f in range(F):
        assert abs(r2[f] / r2[4] - math.exp(-2 * gamma * abs(f - 4))) < 1e-14
    G = sum(math.exp(-2 * gamma * abs(f - 4)) for f in range(F))
    assert abs(math.pi * r2.sum() - 2.0 * math.e) < 1e-9 * G


def _gauss_circle(r2):
    """Lattice points (x, y) with x^2 + y^2 <= r2."""
    R = int(math.isqrt(int(math.floor(r2))))
    return sum(2 * int(math.isqrt(int(math.floor(r2 - x * x)))) + 1 for x in range(-R, R + 1))


def test_kept_count_is_the_gauss_circle_count():
    F, Hh, W = 1, 41, 41
    i = 20 * W + 20  # centre of the frame: no edge clipping
    for H in (0.5, 2.0, 3.7):
        kept, _ = tra_token.key_keep(i, H, F, Hh, W, 1.0, 0.0)
        r2 = math.exp(H) / math.pi
        assert kept.sum() == _gauss_circle(r2)


def _brute_lists(H, F, Hh, W, B, tau, gamma, vote):
    N = F * Hh * W
    nb = (N + B - 1) // B
    S = Hh * W
    out = {}
    for qb in range(nb):
        cnt = [0] * nb
        for i in range(qb * B, min(N, qb * B + B)):
            fi, hi, wi = i // S, (i % S) // W, i % W
            G = sum(math.exp(-2 * gamma * abs(f - fi)) for f in range(F))
            r0sq = tau * math.exp(H[i]) / (math.pi * G)
            for j in range(N):
                fj, hj, wj = j // S, (j % S) // W, j % W
                rf = r0sq * math.exp(-2 * gamma * abs(fj - fi))
                if math.pi * rf >= 1.0 and (hj - hi) ** 2 + (wj - wi) ** 2 <= rf:
                    cnt[j // B] += 1
        out[qb] = [kb for kb in range(nb) if cnt[kb] >= vote]
    return out


def test_block_lists_equal_brute_force():
    rng = np.random.default_rng(3)
    F, Hh, W, B = 3, 5, 7, 16  # N = 105: partial last block
    H = rng.uniform(0.0, 3.0, size=F * Hh * W)
    for vote in (1, 3):
        got = tra_token.block_lists(H, F, Hh, W, B, 1.5, 0.35, vote)
        ref = _brute_lists(H, F, Hh, W, B, 1.5, 0.35, vote)
        for qb in ref:
            ids, amb = got[qb]
            assert set(ids.tolist()) ^ set(ref[qb]) <= set(amb.tolist())
            assert list(ids) == sorted(ids)


def test_huge_budget_keeps_everything():
    F, Hh, W, B = 2, 4, 6, 8
    H = np.zeros(F * Hh * W)
    got = tra_token.block_lists(H, F, Hh, W, B, 1e6, 0.0, 1)
    nb = (F * Hh * W + B - 1) // B
    assert all(list(ids) == list(range(nb)) for ids, _ in got.values())


def test_tiny_budget_keeps_nothing():
    # every frame's share of the budget is below one token
    F, Hh, W, B = 3, 4, 4, 4
    H = np.zeros(F * Hh * W)
    got = tra_token.block_lists(H, F, Hh, W, B, 1e-3, 0.2, 1)
    assert all(len(ids) == 0 and len(amb) == 0 for ids, amb in got.values())


def test_steep_decay_keeps_only_the_query_frame():
    # gamma = 5: the neighbouring frames' shares are e^-10 of the own frame's
    F, Hh, W, B = 3, 6, 6, 6
    N = F * Hh * W
    S = Hh * W
    H = np.full(N, math.log(20.0))  # n = 20 keys, ~all in the own frame
    got = tra_token.block_lists(H, F, Hh, W, B, 1.0, 5.0, 1)
    for qb, (ids, amb) in got.items():
        frames = {int(kb) * B // S for kb in ids}
        assert frames == {qb * B // S} and len(amb) == 0


def test_vote_above_pair_count_is_empty():
    F, Hh, W, B = 2, 3, 3, 6
    H = np.ones(F * Hh * W)
    got = tra_token.block_lists(H, F, Hh, W, B, 1.0, 0.1, vote=10 ** 6)
    assert all(len(ids) == 0 for ids, _ in got.values())


def _nearest_key_lists(H, F, Hh, W, B, tau, gamma):
    """Vote-1 block lists from the nearest key of each grid-row segment: a
    segment [w0, w1] of row (f, h) holds a kept key for query i iff its key
    at column clamp(w_i, w0, w1) is kept (that key minimises the squared
    distance within the row)."""
    N = F * Hh * W
    S = Hh * W
    nb = (N + B - 1) // B
    out = {}
    for qb in range(nb):
        kept = set()
        for i in range(qb * B, min(N, qb * B + B)):
            fi, hi, wi = i // S, (i % S) // W, i % W
            r2 = tra_token.radius2(H[i], fi, F, tau, gamma)
            for kb in range(nb):
                if kb in kept:
                    continue
                t, t1 = kb * B, min(N, kb * B + B)
                while t < t1:
                    f, h, w0 = t // S, (t % S) // W, t % W
                    w1 = min(W - 1, w0 + (t1 - 1 - t))
                    t += w1 - w0 + 1
                    if np.pi * r2[f] < 1.0:
                        continue
                    wn = min(max(wi, w0), w1)
                    if (h - hi) ** 2 + (wn - wi) ** 2 <= r2[f]:
                        kept.add(kb)
                        break
        out[qb] = sorted(kept)
    return out


@pytest.mark.parametrize("tau", [0.1, 0.15])
@pytest.mark.parametrize("F,Hh,W,B,seed", [(3, 5, 7, 16, 0), (4, 6, 9, 32, 1), (2, 7, 5, 8, 2)])
def test_vote_one_equals_nearest_key_of_each_row_segment(F, Hh, W, B, seed, tau):
    # blocks straddle rows and frames (W and S are not multiples of B) and
    # the last block is partial on the first two grids
    N = F * Hh * W
    H = np.random.default_rng(seed).uniform(1.0, 4.0, N)
    gamma = 0.3
    got = tra_token.block_lists(H, F, Hh, W, B, tau, gamma, vote=1)
    ref = _nearest_key_lists(H, F, Hh, W, B, tau, gamma)
    sizes = []
    for qb, (ids, amb) in got.items():
        assert len(amb) == 0
        assert ids.tolist() == ref[qb], qb
        sizes.append(len(ids))
    nb = (N + B - 1) // B
    assert 0 < min(sizes) and max(sizes) < nb  # neither empty nor dense rows


def _rectangles(block_tokens, S, W):
    """Maximal key rectangles of one block: the block's tokens (raster ids,
    in sequence order) cut into runs along grid rows, and runs of
    consecutive rows with the same column range merged (f, h0, h1, w0, w1)."""
    runs = []
    for t in block_tokens:
        f, h, w = t // S, (t % S) // W, t % W
        if runs and runs[-1][:2] == [f, h] and runs[-1][3] == w - 1:
            runs[-1][3] = w
        else:
            runs.append([f, h, w, w])
    rects = []
    for f, h, w0, w1 in runs:
        if rects and rects[-1][0] == f and rects[-1][2] == h - 1 and rects[-1][3:] == [w0, w1]:
            rects[-1][2] = h
        else:
            rects.append([f, h, h, w0, w1])
    return rects


@pytest.mark.parametrize("F,Hh,W,th,tw,B,seed", [(2, 12, 16, 4, 8, 32, 0), (3, 10, 13, 4, 4, 16, 1),
                                                 (2, 9, 20, 3, 20, 24, 2), (2, 8, 8, 1, 8, 16, 3)])
def test_vote_one_equals_nearest_key_of_each_rectangle(F, Hh, W, th, tw, B, seed):
    """With vote 1 a key block is listed iff, for some query of the block, the
    key of one of the block's maximal rectangles nearest to the query
    (row clamp(h_i, h0, h1), column clamp(w_i, w0, w1)) is kept: inside a
    rectangle of one frame that key minimises the squared distance, and the
    frame's share does not depend on the key.  Tile-major orders with ragged
    tiles, blocks that cut tiles, and the raster order (t_h = 1, t_w = W)."""
    N, S = F * Hh * W, Hh * W
    perm = tile_major.order(F, Hh, W, th, tw)
    H = np.random.default_rng(seed).uniform(1.0, 4.0, N)
    tau, gamma = 0.12, 0.3
    got = tra_token.block_lists(H, F, Hh, W, B, tau, gamma, vote=1, perm=perm)
    nb = (N + B - 1) // B
    rects = [_rectangles(perm[kb * B:min(N, kb * B + B)], S, W) for kb in range(nb)]
    sizes = []
    for qb in range(nb):
        kept = set()
        for i in perm[qb * B:min(N, qb * B + B)]:
            fi, hi, wi = i // S, (i % S) // W, i % W
            r2 = tra_token.radius2(H[i], fi, F, tau, gamma)
            for kb in range(nb):
                if kb in kept:
                    continue
                for f, h0, h1, w0, w1 in rects[kb]:
                    if np.pi * r2[f] < 1.0:
                        continue
                    hn, wn = min(max(hi, h0), h1), min(max(wi, w0), w1)
                    if (hn - hi) ** 2 + (wn - wi) ** 2 <= r2[f]:
                        kept.add(kb)
                        break
        ids, amb = got[qb]
        assert len(amb) == 0
        assert ids.tolist() == sorted(kept), qb
        sizes.append(len(ids))
    assert 0 < min(sizes) and max(sizes) < nb


@pytest.mark.parametrize("delta,near", [(1e-5, True), (-1e-5, True), (4e-5, False),
                                        (-4e-5, False)])
def test_near_band_at_the_disk_edge(delta, near):
    """One frame (G = 1, no decay), H = 0: r^2 = tau / pi.  With
    tau = 25 pi (1 + delta) the key at (dh, dw) = (3, 4) sits at d^2 = 25, a
    relative distance |delta| / (1 + delta) from the disk edge: near within
    2.5e-5, kept iff delta >= 0."""
    F, Hh, W = 1, 11, 11
    i = 5 * W + 5                                   # the centre token
    tau = 25.0 * math.pi * (1.0 + delta)
    kept, nr = tra_token.key_keep(i, 0.0, F, Hh, W, tau, 0.25)
    j = (5 + 3) * W + (5 + 4)
    assert bool(kept[j]) == (delta > 0)
    assert bool(nr[j]) == near
    # keys one unit of d^2 away are far from the edge
    for j2 in ((5 + 5) * W + 5 - 1, 5 * W + 5 + 4):  # d^2 = 26 and 16
        assert not nr[j2]


@pytest.mark.parametrize("delta,near", [(1e-5, True), (-1e-5, True), (4e-5, False),
                                        (-4e-5, False)])
def test_near_band_at_one_token_share(delta, near):
    """One frame, H = 0, tau = 1 + delta: the frame's share is n_f = tau
    tokens.  The query's own key (d^2 = 0, far inside the disk) is kept iff
    n_f >= 1, and near iff n_f is within 2.5e-5 of one token."""
    F, Hh, W = 1, 5, 5
    i = 12
    kept, nr = tra_token.key_keep(i, 0.0, F, Hh, W, 1.0 + delta, 0.25)
    assert bool(kept[i]) == (delta > 0)
    assert bool(nr[i]) == near
