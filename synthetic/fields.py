"""Smooth random Fourier fields plus noise: the seeded Q/K/V recipe.

For a token at grid position (f, h, w) with normalised coordinates
x = (f/F, h/H, w/W), one field is

    X(x) = sum_{m=1..8} a_m * cos(2*pi * k_m . x + phi_m)        (a d-vector)

with integer wave vectors k_m in {0..3}^3, phases phi_m ~ U[0, 2*pi)^d and
amplitudes a_m ~ N(0, 1/8)^d.  Every head of Q, K and V draws its own modes.
Noise N(0, sigma^2) is added per element; sigma is either constant or drawn
per 128-token block ("per-region" noise, shared by heads and by Q/K/V).
Q and K are then multiplied by one common factor so that q.k/sqrt(d) over
random same-head token pairs has the requested standard deviation.

The cosine of a sum is expanded as cos(p)cos(phi) - sin(p)sin(phi), so the
field is two small matrix products [N, 8] x [8, d] instead of N*d*8 cosines.
"""
import numpy as np
import torch

N_MODES = 8
K_MAX = 3
N_LOGIT_PAIRS = 20000
NOISE_REGION = 128


def _normalised_coords(F, H, W):
    t = np.arange(F * H * W, dtype=np.int64)
    S = H * W
    f = t // S
    h = (t % S) // W
    w = t % W
    return np.stack([f / F, h / H, w / W], axis=1)  # [N, 3] float64


def _one_field(rng, x, d):
    k = rng.integers(0, K_MAX + 1, size=(N_MODES, 3)).astype(np.float64)
    phi = rng.uniform(0.0, 2.0 * np.pi, size=(N_MODES, d))
    a = rng.normal(0.0, np.sqrt(1.0 / N_MODES), size=(N_MODES, d))
    phase = 2.0 * np.pi * (x @ k.T)  # [N, 8]
    return np.cos(phase) @ (a * np.cos(phi)) - np.sin(phase) @ (a * np.sin(phi))


def _streams(seed):
    ss = np.random.SeedSequence(seed)
    q, k, v, diff, region, pairs = ss.spawn(6)
    return dict(q=np.random.default_rng(q), k=np.random.default_rng(k),
                v=np.random.default_rng(v), diff=np.random.default_rng(diff),
                region=np.random.default_rng(region),
                pairs=np.random.default_rng(pairs))


def _noise_sigma(w, rng_region):
    """Per-token noise std [N] (float32) or a scalar."""
    N = w["F"] * w["H"] * w["W"]
    if w.get("noise_block"):
        lo, hi = w["noise_block"]
        n_reg = (N + NOISE_REGION - 1) // NOISE_REGION
        sig = lo + (hi - lo) * rng_region.random(n_reg)
        return np.repeat(sig, NOISE_REGION)[:N].astype(np.float32)[:, None]
    return np.float32(w["noise"])


def make_qkv(w, out_dtype=None):
    """Return CPU tensors q, k, v of shape [heads, N, d].

    The element type is the workload's ("f32" -> float32, "bf16" ->
    bfloat16, rounded to nearest even from the fp32 field) unless out_dtype
    is given.  Deterministic in w["seed"].
    """
    heads, F, H, W, d = w["heads"], w["F"], w["H"], w["W"], w["d"]
    N = F * H * W
    st = _streams(w["seed"])
    x = _normalised_coords(F, H, W)
    sigma = _noise_sigma(w, st["region"])
    noise_buf = np.empty((N, d), np.float32)
    arrs = {}
    for name in ("q", "k", "v"):
        rng = st[name]
        arr = np.empty((heads, N, d), np.float32)
        for h in range(heads):
            arr[h] = _one_field(rng, x, d)
            rng.standard_normal(out=noise_buf, dtype=np.float32)
            arr[h] += noise_buf * sigma
        arrs[name] = arr
    if w.get("logit_std"):
        rng = st["pairs"]
        hh = rng.integers(0, heads, N_LOGIT_PAIRS)
        ii = rng.integers(0, N, N_LOGIT_PAIRS)
        jj = rng.integers(0, N, N_LOGIT_PAIRS)
        qs = arrs["q"][hh, ii].astype(np.float64)
        ks = arrs["k"][hh, jj].astype(np.float64)
        logits = (qs * ks).sum(1) / np.sqrt(d)
        c = np.float32(np.sqrt(w["logit_std"] / logits.std()))
        arrs["q"] *= c
        arrs["k"] *= c
    if out_dtype is None:
        out_dtype = torch.float32 if w["dtype"] == "f32" else torch.bfloat16
    return tuple(torch.from_numpy(arrs[n]).to(out_dtype) for n in ("q", "k", "v"))


def make_difficulty(w):
    """Per-token difficulty score ~ Beta(2, 5), float32 [N] (shared by heads)."""
    N = w["F"] * w["H"] * w["W"]
    st = _streams(w["seed"])
    return st["diff"].beta(2.0, 5.0, size=N).astype(np.float32)
