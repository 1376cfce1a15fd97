"""Token grid geometry (oracle side).

Tokens of a video latent of F frames x H x W are numbered in raster order,
frame-major: t = f*S + h*W + w with S = H*W.  "Dense 3D self-attention over
F*H*W tokens" ("Token Radius Attention for Efficient Video Generation",
1. Problem Statement) fixes the token set; raster order is the reading of a
[heads, F*H*W, d] tensor.

Block b covers tokens [b*B, min((b+1)*B, N)); the last block may be partial.
"""
import numpy as np


def coords(t, F, H, W):
    """(f, h, w) of token index t (scalar or array)."""
    S = H * W
    t = np.asarray(t)
    return t // S, (t % S) // W, t % W


def n_blocks(N, B):
    return (N + B - 1) // B


def block_range(b, B, N):
    """Half-open token range of block b."""
    return b * B, min((b + 1) * B, N)


def block_len(b, B, N):
    lo, hi = block_range(b, B, N)
    return hi - lo


def block_frame_intervals(b, B, N, S):
    """Split block b into per-frame runs: list of (f, s_lo, s_hi), inclusive
    spatial (flattened h*W+w) bounds inside frame f."""
    t0, t1 = block_range(b, B, N)
    out = []
    t = t0
    while t < t1:
        f = t // S
        end = min(t1, (f + 1) * S)  # exclusive
        out.append((f, t - f * S, end - 1 - f * S))
        t = end
    return out


def unit_tokens(units, U, N):
    """Concatenated token ids of KV units (U tokens each, clipped at N)."""
    if len(units) == 0:
        return np.zeros(0, dtype=np.int64)
    parts = [np.arange(u * U, min((u + 1) * U, N), dtype=np.int64) for u in units]
    return np.concatenate(parts)
