"""Workload table: grid shapes, input recipe and selector parameters.

Each entry is a plain dictionary of constants.  Grid shapes follow the latent
grids of the video models the pages evaluate (Wan2.1-1.3B, Wan2.2-5B,
HunyuanVideo); the parameters are the ones each workload states, plus the
readings recorded beside them.

Keys
----
heads, F, H, W, d   problem shape; N = F*H*W tokens per head, raster order.
dtype               "f32" or "bf16": element type handed to the library.
noise               iid noise std added to every element, or None.
noise_block         (lo, hi): per 128-token block the noise std is drawn
                    uniformly from [lo, hi) instead ("per-region" noise).
logit_std           Q and K share one scale factor chosen so that the std of
                    q.k/sqrt(d) over random same-head pairs is this value.
block_q, kv_unit    query block and key/value unit in tokens.
selector            "radial" | "entropy" | "ibcs_sip" | "routed" | "tra_token" |
                    "dynrad".
layout              optional (t_h, t_w): the token-level pipeline runs in the
                    tile-major token order with t_h x t_w spatial tiles
                    (q, k, v permuted in, o permuted back); absent = raster.
"""
import copy

WORKLOADS = {
    # 1 head, 4 frames of 8x8 latents, d=64, fp32 inputs.  Radial mask with
    # 64-token blocks: full attention within |df| <= 1, window halving for each
    # doubling of |df| beyond that.  With 64-token blocks every block pair
    # keeps at least one token pair, so the result must equal dense attention.
    "tiny_radial": dict(
        heads=1, F=4, H=8, W=8, d=64, dtype="f32", noise=0.5, noise_block=None,
        logit_std=None, block_q=64, kv_unit=64, selector="radial",
        radial=dict(w0=64, w_off=0, full_df=1), seed=0),
    # Same grid with 16-token blocks: the block mask is no longer full.
    "tiny_radial_b16": dict(
        heads=1, F=4, H=8, W=8, d=64, dtype="f32", noise=0.5, noise_block=None,
        logit_std=None, block_q=16, kv_unit=16, selector="radial",
        radial=dict(w0=64, w_off=0, full_df=1), seed=0),
    # Wan2.1-1.3B latent grid 21x30x52 (N=32760), 12 heads, d=128, bf16.
    # Window at frame distance df is (30*52) / 2^floor(log2(1+df)) tokens.
    "wan_radial": dict(
        heads=12, F=21, H=30, W=52, d=128, dtype="bf16", noise=0.5,
        noise_block=None, logit_std=3.0, block_q=128, kv_unit=128,
        selector="radial", radial=dict(w0=1560, w_off=1, full_df=-1), seed=0),
    # Entropy -> radius at the Wan2.1-1.3B shape.  Per-region noise std in
    # [0.2, 2.0).  alpha/beta map the 5th..95th percentile of the pooled
    # entropies onto radii 1..2 (fixed once from the oracle's entropies by
    # tests/golden/make_entropy_calibration.py; values stored in
    # tests/golden/entropy_calibration.json and copied here).
    "tra_entropy": dict(
        heads=12, F=21, H=30, W=52, d=128, dtype="bf16", noise=None,
        noise_block=(0.2, 2.0), logit_std=3.0, block_q=128, kv_unit=128,
        selector="entropy",
        entropy=dict(alpha=-208.83056640625, beta=38.206417083740234, r_lo=1, r_hi=2,
                     tile_h=8, tile_w=16),
        seed=0),
    # Token-level TRA pipeline at the Wan2.1-1.3B shape: per-query entropy
    # from a dense warm-up, budget tau*exp(H), a disk per frame whose radius
    # decays by exp(-gamma*delta) with frame distance, token voting into
    # 128-token block lists.  tau is fixed once from the oracle so that the
    # blocks keep about 14% of the key blocks, inside the 9-19% the pages
    # report (tests/golden/make_tra_token_calibration.py; value stored in
    # tests/golden/tra_token_calibration.json and copied here).
    "tra_token": dict(
        heads=12, F=21, H=30, W=52, d=128, dtype="bf16", noise=0.5,
        noise_block=None, logit_std=3.0, block_q=128, kv_unit=128,
        selector="tra_token", tra_token=dict(tau=0.07146470248699188, gamma=0.25, vote=1),
        seed=0),
    # The token-level TRA pipeline in a tile-major token order on a wide grid
    # (13 latent frames x 40 x 128, N = 66,560), where a 128-token raster
    # block is a single grid row and the oracle keeps fewer block pairs with
    # 16 x 8 spatial tiles (10.5% of the pairs of 24 seeded query blocks)
    # than in raster order (12.9%).  Same tau, gamma and vote as tra_token.
    "tra_token_tiled": dict(
        heads=12, F=13, H=40, W=128, d=128, dtype="bf16", noise=0.5,
        noise_block=None, logit_std=3.0, block_q=128, kv_unit=128,
        selector="tra_token", tra_token=dict(tau=0.07146470248699188, gamma=0.25, vote=1),
        layout=(16, 8), seed=0),
    # DynamicRad-style selection inside the radial prior at the Wan2.1-1.3B
    # shape (the wan_radial lists are the candidates): static ratio keeps the
    # best 35% of each row's candidates by pooled attention probability,
    # dynamic threshold the shortest best-first prefix holding 35% of the
    # mass; both leave about 80% of all block pairs out (the page reports
    # over 80% effective sparsity).
    "dynrad_static": dict(
        heads=12, F=21, H=30, W=52, d=128, dtype="bf16", noise=0.5,
        noise_block=None, logit_std=3.0, block_q=128, kv_unit=128, selector="dynrad",
        radial=dict(w0=1560, w_off=1, full_df=-1), dynrad=dict(mode="static", ratio=0.35),
        seed=0),
    "dynrad_dynamic": dict(
        heads=12, F=21, H=30, W=52, d=128, dtype="bf16", noise=0.5,
        noise_block=None, logit_std=3.0, block_q=128, kv_unit=128, selector="dynrad",
        radial=dict(w0=1560, w_off=1, full_df=-1), dynrad=dict(mode="dynamic", threshold=0.35),
        seed=0),
    # HetA-style routing at the Wan2.2-5B shape 31x44x80 (N=109120), 24 heads.
    # Top 20% of tokens by a Beta(2,5) difficulty go to dense attention; the
    # rest use a local window of +-1 frame x 16x16 tokens.
    "heta_routed": dict(
        heads=24, F=31, H=44, W=80, d=128, dtype="bf16", noise=0.5,
        noise_block=None, logit_std=3.0, block_q=128, kv_unit=16,
        selector="routed",
        routed=dict(dense_frac=0.2, win_f=1, win_h=8, win_w=8), seed=0),
    # AB-style importance sampling at the HunyuanVideo shape 33x45x80
    # (N=118800), 24 heads: k-means k=4 x 5 iterations per 128-query block
    # against 16-key sub-block means, ~10% of sub-blocks drawn per query
    # block with probability proportional to importance, weights 1/pi.
    "ab_sampled": dict(
        heads=24, F=33, H=45, W=80, d=128, dtype="bf16", noise=0.5,
        noise_block=None, logit_std=3.0, block_q=128, kv_unit=16,
        selector="ibcs_sip",
        ibcs=dict(k=4, iters=5, sample_frac=0.10, seed=0x5EED5A3C1E5B00B5),
        seed=0),
}


def workload(name, **overrides):
    """Return a deep copy of a workload entry with top-level overrides applied.

    Overriding F/H/W/heads gives the reduced grids the tests use; the input
    recipe and selector parameters stay the same.
    """
    w = copy.deepcopy(WORKLOADS[name])
    w.update(overrides)
    w["name"] = name
    w["N"] = w["F"] * w["H"] * w["W"]
    return w
