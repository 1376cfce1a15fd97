"""The seeded input recipe: deterministic, right shapes, logit scale."""
import numpy as np
import torch

from synthetic import make_difficulty, make_qkv, workload


def test_deterministic_and_shapes():
    w = workload("tiny_radial")
    a = make_qkv(w)
    b = make_qkv(w)
    for x, y in zip(a, b):
        assert x.shape == (1, 256, 64) and x.dtype == torch.float32
        assert torch.equal(x, y)
    assert not torch.equal(a[0], a[1])


def test_logit_std_and_bf16():
    w = workload("wan_radial", heads=2, F=3, H=6, W=10)
    q, k, v = make_qkv(w)
    assert q.dtype == torch.bfloat16 and q.shape == (2, 180, 128)
    s = torch.einsum("hnd,hmd->hnm", q.double(), k.double()) / np.sqrt(128)
    assert 2.0 < float(s.std()) < 4.0


def test_region_noise_and_difficulty():
    w = workload("tra_entropy", heads=1, F=2, H=8, W=16)
    q, _, _ = make_qkv(w)
    assert q.shape == (1, 256, 128)
    d = make_difficulty(workload("heta_routed", F=2, H=4, W=8))
    assert d.dtype == np.float32 and d.shape == (64,) and 0 < d.min() and d.max() < 1


def test_entropy_workload_uses_the_stored_calibration():
    import json
    import os
    from synthetic import workload
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                        "entropy_calibration.json")
    cal = json.load(open(path))
    e = workload("tra_entropy")["entropy"]
    assert (e["alpha"], e["beta"], e["r_lo"], e["r_hi"]) == (cal["alpha"], cal["beta"],
                                                             cal["r_lo"], cal["r_hi"])
