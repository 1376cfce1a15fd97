"""GPU parity of the DynamicRad dual-mode selector ("DynamicRad: Content-
Adaptive Sparse Attention for Long Video Diffusion", Abstract: selection
inside a radial prior by static ratio or dynamic threshold) and of the
attention over its lists.

Lists must equal the fp64 oracle bit-exactly, except rows the oracle flags
as near a decision (two candidates whose order decides membership within
1e-5 relative, or a prefix mass within 1e-5 of the threshold), which are
counted and bounded."""
import numpy as np
import pytest
import torch

from oracle import dynrad
from oracle.pipeline import block_sparse_rows
from synthetic import make_qkv, workload
from tests._util import assert_close_attn

pytestmark = pytest.mark.gpu


def _run(w, qd, kd):
    from sparse_spatiotemporal_attention_video_b200 import api, session
    L = session.Lists(w)
    ws = session.selector_workspace(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_build_blocks(session.problem(w), session.selector(w), qd, kd, L.struct, workspace=ws,
                         dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, api.sta_dev_status_string(int(st.item()))
    return L


def _check(w, L, q, k, heads, qblocks=None):
    c = w["dynrad"]
    nqb = (w["N"] + w["block_q"] - 1) // w["block_q"]
    rows = L.host_rows()
    near = checked = 0
    for h in heads:
        ref = dynrad.select(q[h].float().numpy().astype(np.float64),
                            k[h].float().numpy().astype(np.float64), w["F"], w["H"], w["W"],
                            w["block_q"], w["radial"], c["mode"], c.get("ratio"),
                            c.get("threshold"))
        for b in (range(nqb) if qblocks is None else qblocks):
            ids, is_near = ref[b]
            if is_near:
                near += 1
                continue
            assert rows[h * nqb + b] == list(ids), (h, b)
            checked += 1
    return checked, near


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("mode,param", [("static", 0.35), ("static", 0.8), ("dynamic", 0.35),
                                        ("dynamic", 0.9)])
def test_small_grid_every_row(cuda_ok, mode, param, d):
    # 6 x 10 x 26 = 1560 tokens: 13 blocks, the last one partial (24 tokens);
    # d = 128 and d = 64 take the 4- and 2-floats-per-lane score paths
    w = workload("dynrad_static", F=6, H=10, W=26, heads=2, d=d)
    w["radial"] = dict(w0=260, w_off=1, full_df=-1)
    w["dynrad"] = dict(mode=mode, **({"ratio": param} if mode == "static" else
                                     {"threshold": param}))
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    L = _run(w, qd, kd)
    checked, near = _check(w, L, q, k, (0, 1))
    assert checked >= 24 and near <= 2
    # attention over the selected blocks
    from sparse_spatiotemporal_attention_video_b200 import api, session
    o = torch.full_like(qd, float("nan"))
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), qd, kd, vd, L.struct, o)
    torch.cuda.synchronize()
    rows = L.host_rows()
    nqb = 13
    for h in (0, 1):
        for b in range(nqb):
            lo, hi = b * 128, min(w["N"], b * 128 + 128)
            ref = block_sparse_rows(q[h], k[h], v[h], b, rows[h * nqb + b], 128, 128)
            assert_close_attn(o[h, lo:hi].float().cpu().numpy(), ref, f"{mode} head {h} qb {b}")


@pytest.mark.parametrize("name", ["dynrad_static", "dynrad_dynamic"])
def test_full_wan_shape_sampled_rows(cuda_ok, name):
    w = workload(name)
    q, k, _ = make_qkv(w)
    L = _run(w, q.cuda(), k.cuda())
    nqb = (w["N"] + 127) // 128
    checked, near = _check(w, L, q, k, (0, 7, 11), [0, 31, 128, 200, nqb - 1])
    assert checked >= 13 and near <= 2
    # about 80% of all block pairs left out
    kept = L.cnt.float().sum().item() / (w["heads"] * nqb * nqb)
    assert 0.12 <= kept <= 0.30, kept
