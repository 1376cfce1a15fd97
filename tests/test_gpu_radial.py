"""GPU parity: static radial selector lists (bit-exact) and radial sparse
attention vs the fp64 oracle on the tiny grid and the Wan2.1-1.3B grid."""
import numpy as np
import pytest
import torch

from oracle import radial
from oracle.pipeline import block_sparse_rows, dense_rows
from synthetic import make_qkv, workload
from tests._util import assert_close_attn

pytestmark = pytest.mark.gpu


def _lib():
    from sparse_spatiotemporal_attention_video_b200 import api, session
    return api, session


def _build(w):
    api, session = _lib()
    L = session.Lists(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_build_blocks(session.problem(w), session.selector(w), None, None, L.struct,
                         dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return L


@pytest.mark.parametrize("name,F,H,W", [
    ("tiny_radial", 4, 8, 8), ("tiny_radial_b16", 4, 8, 8),
    ("wan_radial", 21, 30, 52),
    ("wan_radial", 5, 7, 9)])      # ragged: N = 315, blocks straddle frames
def test_radial_lists_bit_exact(cuda_ok, name, F, H, W):
    w = workload(name, F=F, H=H, W=W)
    if w["F"] == 5:
        w["radial"] = dict(w0=63, w_off=1, full_df=-1)
        w["block_q"] = w["kv_unit"] = 16
    L = _build(w)
    got = L.host_rows()
    ref = radial.block_lists(w["F"], w["H"], w["W"], w["block_q"], w["radial"])
    assert len(got) == len(ref)
    for qb, (a, b) in enumerate(zip(got, ref)):
        assert a == list(b), f"row {qb}"
    assert int(L.required_cap.item()) == max(len(r) for r in ref)


@pytest.mark.parametrize("name", ["tiny_radial", "tiny_radial_b16"])
def test_tiny_radial_attention_whole(cuda_ok, name):
    api, session = _lib()
    w = workload(name)
    q, k, v = make_qkv(w)
    L = _build(w)
    prob = session.problem(w)
    ws = torch.empty(api.sta_attn_workspace(prob), dtype=torch.uint8, device="cuda")
    o = torch.full_like(q, float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(prob, session.attn_params(w), q.cuda(), k.cuda(), v.cuda(), L.struct,
                            o, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    lists = radial.block_lists(w["F"], w["H"], w["W"], w["block_q"], w["radial"])
    ref = np.concatenate([block_sparse_rows(q[0], k[0], v[0], qb, lists[qb], w["block_q"],
                                            w["kv_unit"]) for qb in range(len(lists))])
    assert_close_attn(o[0].cpu().numpy(), ref, name)
    if name == "tiny_radial":
        # 64-token blocks keep every pair: the result is dense attention
        dense = np.concatenate([dense_rows(q[0], k[0], v[0], qb, 64) for qb in range(4)])
        assert_close_attn(o[0].cpu().numpy(), dense, "tiny radial vs dense")


def test_wan_radial_attention_sampled_blocks(cuda_ok):
    api, session = _lib()
    w = workload("wan_radial")
    q, k, v = make_qkv(w)
    L = _build(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), qd, kd, vd, L.struct, o,
                            dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    lists = radial.block_lists(w["F"], w["H"], w["W"], 128, w["radial"])
    nqb = len(lists)
    rng = np.random.default_rng(1)
    blocks = sorted({0, nqb - 1, *rng.choice(np.arange(1, nqb - 1), 14, replace=False).tolist()})
    oc = o.cpu()
    for h in range(w["heads"]):
        for qb in blocks:
            ref = block_sparse_rows(q[h], k[h], v[h], qb, lists[qb], 128, 128)
            got = oc[h, qb * 128: qb * 128 + ref.shape[0]].float().numpy()
            assert_close_attn(got, ref, f"head {h} qblock {qb}")
