"""GPU parity of the attention kernel on seeded random lists: every supported
head dim and unit size, ragged tails, empty rows, log-weights, the dense
path, and invariance to the contents of unkept keys."""
import math

import numpy as np
import pytest
import torch

from oracle.pipeline import block_sparse_rows, dense_rows
from synthetic import make_qkv, workload
from tests._util import assert_close_attn

pytestmark = pytest.mark.gpu


def _mods():
    from sparse_spatiotemporal_attention_video_b200 import api, session
    from sparse_spatiotemporal_attention_video_b200._lib import (AttnParams, BlockLists, Problem,
                                                                STA_ATTN_LISTS)
    return api, session, AttnParams, BlockLists, Problem, STA_ATTN_LISTS


def _random_lists(rng, rows, n_units, cap, empty_rows=(), full_rows=()):
    idx = np.zeros((rows, cap), np.int32)
    cnt = np.zeros(rows, np.int32)
    lists = []
    for r in range(rows):
        if r in empty_rows:
            sel = np.zeros(0, np.int64)
        elif r in full_rows:
            sel = np.arange(min(n_units, cap))
        else:
            m = int(rng.integers(1, min(n_units, cap) + 1))
            sel = np.sort(rng.choice(n_units, m, replace=False))
        idx[r, :len(sel)] = sel
        cnt[r] = len(sel)
        lists.append(sel)
    return idx, cnt, lists


def _run(w, q, k, v, idx, cnt, cap, logw=None, head_shared=False):
    api, session, AttnParams, BlockLists, Problem, STA_ATTN_LISTS = _mods()
    prob = session.problem(w)
    prm = AttnParams()
    prm.mode, prm.block_q, prm.kv_unit, prm.scale = STA_ATTN_LISTS, w["block_q"], w["kv_unit"], 0.0
    di = torch.from_numpy(idx).cuda()
    dc = torch.from_numpy(cnt).cuda()
    dl = torch.from_numpy(logw).cuda() if logw is not None else None
    L = BlockLists()
    L.idx, L.cnt, L.cap, L.head_shared = di.data_ptr(), dc.data_ptr(), cap, int(head_shared)
    L.logw = dl.data_ptr() if dl is not None else None
    ws = torch.empty(max(1, api.sta_attn_workspace(prob)), dtype=torch.uint8, device="cuda")
    o = torch.full(q.shape, float("nan"), dtype=q.dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(prob, prm, q.cuda(), k.cuda(), v.cuda(), L, o, workspace=ws,
                            dev_status=st)
    torch.cuda.synchronize()
    return o.cpu(), int(st.item())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("unit", [16, 32, 64, 128])
def test_random_lists_match_oracle(cuda_ok, d, unit):
    # 3 frames of 10x13: N = 390 = 3*128 + 6 (ragged last query block and unit)
    w = workload("wan_radial", heads=2, F=3, H=10, W=13, d=d, block_q=128, kv_unit=unit)
    q, k, v = make_qkv(w)
    N = w["N"]
    nqb = (N + 127) // 128
    n_units = (N + unit - 1) // unit
    rng = np.random.default_rng(d * 1000 + unit)
    cap = n_units
    idx, cnt, lists = _random_lists(rng, 2 * nqb, n_units, cap, empty_rows=(1,),
                                    full_rows=(2,))
    o, st = _run(w, q, k, v, idx, cnt, cap)
    assert st & 0x4  # the empty row is reported
    for h in range(2):
        for qb in range(nqb):
            r = h * nqb + qb
            lo, hi = qb * 128, min(N, qb * 128 + 128)
            got = o[h, lo:hi].float().numpy()
            if len(lists[r]) == 0:
                assert np.all(got == 0)
                continue
            ref = block_sparse_rows(q[h], k[h], v[h], qb, lists[r], 128, unit)
            assert_close_attn(got, ref, f"d={d} unit={unit} head {h} qb {qb}")


def test_log_weights_match_oracle(cuda_ok):
    w = workload("ab_sampled", heads=2, F=4, H=9, W=16, kv_unit=16)
    q, k, v = make_qkv(w)
    N = w["N"]
    nqb = (N + 127) // 128
    n_units = N // 16
    rng = np.random.default_rng(7)
    idx, cnt, lists = _random_lists(rng, 2 * nqb, n_units, 64)
    logw = np.zeros(idx.shape, np.float32)
    for r, l in enumerate(lists):
        logw[r, :len(l)] = -np.log(rng.uniform(0.02, 1.0, len(l)))
    o, st = _run(w, q, k, v, idx, cnt, 64, logw=logw)
    assert st == 0
    for h in range(2):
        for qb in range(nqb):
            r = h * nqb + qb
            ref = block_sparse_rows(q[h], k[h], v[h], qb, lists[r], 128, 16, logw[r, :len(lists[r])])
            got = o[h, qb * 128: min(N, qb * 128 + 128)].float().numpy()
            assert_close_attn(got, ref, f"weighted head {h} qb {qb}")


def test_unkept_keys_do_not_matter(cuda_ok):
    w = workload("wan_radial", heads=1, F=2, H=16, W=16, kv_unit=32)
    q, k, v = make_qkv(w)
    N = w["N"]
    rng = np.random.default_rng(3)
    idx, cnt, lists = _random_lists(rng, 4, N // 32, N // 32)
    o1, _ = _run(w, q, k, v, idx, cnt, N // 32)
    kept = np.zeros(N, bool)
    for l in lists:
        for u in l:
            kept[u * 32:(u + 1) * 32] = True
    # unkept keys are unused by every row only if no row keeps them
    k2, v2 = k.clone(), v.clone()
    noise = torch.from_numpy(rng.normal(size=(int((~kept).sum()), 128)) * 50).to(k.dtype)
    k2[0, torch.from_numpy(~kept)] = noise
    v2[0, torch.from_numpy(~kept)] = noise * 3
    o2, _ = _run(w, q, k2, v2, idx, cnt, N // 32)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("d,F,H,W", [(128, 3, 10, 13), (64, 4, 8, 8), (128, 2, 16, 20)])
def test_dense_path_matches_oracle(cuda_ok, d, F, H, W):
    api, session, *_ = _mods()
    w = workload("wan_radial", heads=2, F=F, H=H, W=W, d=d)
    q, k, v = make_qkv(w)
    o = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_dense_attn_fwd(session.problem(w), q.cuda(), k.cuda(), v.cuda(), 0.0, o,
                           dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    N = w["N"]
    oc = o.cpu()
    for h in range(2):
        ref = np.concatenate([dense_rows(q[h], k[h], v[h], qb, 128)
                              for qb in range((N + 127) // 128)])
        assert_close_attn(oc[h].float().numpy(), ref, f"dense d={d} head {h}")


def test_dense_matches_torch_sdpa_at_wan_shape(cuda_ok):
    """Whole Wan2.1-1.3B grid: the dense path against torch's SDPA (fp32
    math on the same bf16 inputs) on one head, as an independent check at
    full sequence length."""
    api, session, *_ = _mods()
    w = workload("wan_radial")
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    api.sta_dense_attn_fwd(session.problem(w), qd, kd, vd, 0.0, o)
    torch.cuda.synchronize()
    for h in (0, 11):
        ref = torch.nn.functional.scaled_dot_product_attention(
            qd[h:h + 1].float(), kd[h:h + 1].float(), vd[h:h + 1].float())[0]
        assert_close_attn(o[h].float().cpu().numpy(), ref.cpu().numpy(), f"sdpa head {h}")
