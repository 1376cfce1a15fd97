"""Error bound of the cubic 2^x the attention kernel evaluates on the FMA
pipe for part of the softmax exponentials.  The coefficients are read from
the kernel header and the kernel's exact fp32 operation sequence is replayed
in numpy (round-to-nearest fp32 at every step)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "sparse_spatiotemporal_attention_video_b200", "csrc", "sm100.cuh")


def _coeffs():
    txt = open(HDR).read()
    m = re.search(r"c0 = ([0-9.e-]+)f, c1 = ([0-9.e-]+)f, c2 = ([0-9.e-]+)f, c3 = ([0-9.e-]+)f", txt)
    return [np.float32(float(g)) for g in m.groups()]


def _replay(x):
    c0, c1, c2, c3 = _coeffs()
    f32 = np.float32
    x = np.maximum(x.astype(np.float32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(np.float32)
    j = (t - f32(12582912.0)).astype(np.float32)
    f = (x - j).astype(np.float32)
    # fmaf = one rounding: evaluate in float64 then round
    f64 = f.astype(np.float64)
    p = (np.float64(c3) * f64 + np.float64(c2)).astype(np.float32)
    p = (p.astype(np.float64) * f64 + np.float64(c1)).astype(np.float32)
    p = (p.astype(np.float64) * f64 + np.float64(c0)).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound_over_the_softmax_range():
    x = np.linspace(-60.0, 8.0, 2_000_001).astype(np.float32)
    got = _replay(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    # far below half an ulp of bf16 (2^-9), where P is rounded anyway
    assert rel.max() < 1.2e-4


def test_integers_and_half_integers():
    for x in [-20.0, -3.5, -1.0, -0.5, 0.0, 0.5, 1.0, 7.5, 8.0]:
        got = float(_replay(np.array([x]))[0])
        assert abs(got / 2.0 ** x - 1.0) < 1.2e-4, x
