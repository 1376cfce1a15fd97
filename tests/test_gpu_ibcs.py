"""GPU parity of the clustering-importance selector with Philox inclusion-
probability sampling, and of the weighted attention over its sub-block lists.

Sampled ids must match the fp64 oracle bit-exactly except (a) entries whose
uniform draw lies within 1e-5 of their inclusion probability and (b) rows
whose k-means had a near-tie assignment (relative margin <= 1e-5); both are
counted and reported separately.  log-weights agree to fp32 accuracy."""
import numpy as np
import pytest
import torch

from oracle import ibcs_sip
from oracle.pipeline import block_sparse_rows, dense_rows
from synthetic import make_qkv, workload
from tests._util import assert_close_attn

pytestmark = pytest.mark.gpu


def _lib():
    from sparse_spatiotemporal_attention_video_b200 import api, session
    return api, session


def _gpu_select(w, qd, kd):
    api, session = _lib()
    L = session.Lists(w)
    ws = session.selector_workspace(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_build_blocks(session.problem(w), session.selector(w), qd, kd, L.struct, workspace=ws,
                         dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, api.sta_dev_status_string(int(st.item()))
    return L


def _check_rows(w, L, q, k, heads, qblocks):
    c = w["ibcs"]
    nqb = (w["N"] + w["block_q"] - 1) // w["block_q"]
    rows = L.host_rows()
    lw = L.logw.cpu().numpy()
    skipped_rows = near_items = checked = 0
    for h in heads:
        ref = ibcs_sip.select(q[h].float().numpy(), k[h].float().numpy(), w["block_q"],
                              w["kv_unit"], c["seed"], h, c["iters"], c["k"], c["sample_frac"],
                              qblocks=qblocks)
        for qb, r in ref.items():
            if r["margin"] <= ibcs_sip.NEAR_THRESHOLD:
                skipped_rows += 1
                continue
            row = h * nqb + qb
            got = rows[row]
            assert got == sorted(got)
            diff = set(got) ^ set(r["ids"].tolist())
            assert diff <= set(r["near_ids"].tolist()), f"head {h} qb {qb}: {sorted(diff)[:8]}"
            near_items += len(diff)
            ref_lw = dict(zip(r["ids"].tolist(), r["logw"].tolist()))
            for pos, j in enumerate(got):
                if j in ref_lw:
                    assert abs(lw[row, pos] - ref_lw[j]) <= 1e-4 * max(1.0, abs(ref_lw[j])), \
                        (h, qb, j, lw[row, pos], ref_lw[j])
            checked += 1
    return checked, skipped_rows, near_items


@pytest.mark.parametrize("F,H,W,frac", [(4, 9, 16, 0.10), (3, 10, 13, 0.25), (2, 16, 16, 0.5)])
def test_ibcs_small_grids_every_row(cuda_ok, F, H, W, frac):
    w = workload("ab_sampled", heads=2, F=F, H=H, W=W)
    w["ibcs"]["sample_frac"] = frac
    q, k, _ = make_qkv(w)
    L = _gpu_select(w, q.cuda(), k.cuda())
    checked, skipped, near = _check_rows(w, L, q, k, (0, 1), None)
    assert checked >= 1 and skipped <= 1 and near <= 2


@pytest.fixture(scope="module")
def hunyuan(cuda_ok):
    """The full HunyuanVideo-shape workload (24 heads x 33x45x80 tokens x 128,
    bf16) on the device with its GPU lists, shared by the full-size tests."""
    w = workload("ab_sampled")
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    L = _gpu_select(w, qd, kd)
    nqb = (w["N"] + 127) // 128
    rng = np.random.default_rng(2)
    qblocks = [0, nqb - 1] + sorted((rng.choice(nqb - 2, 6, replace=False) + 1).tolist())
    yield dict(w=w, q=q, k=k, v=v, qd=qd, kd=kd, vd=vd, L=L, qblocks=qblocks)
    del qd, kd, vd
    torch.cuda.empty_cache()


def test_ibcs_full_hunyuan_shape_sampled_rows(hunyuan):
    w, q, k, L, qblocks = (hunyuan[x] for x in ("w", "q", "k", "L", "qblocks"))
    checked, skipped, near = _check_rows(w, L, q, k, (0, 13, 23), qblocks)
    assert checked >= 20 and skipped <= 2 and near <= 4
    # about 10% of the sub-blocks are kept per row
    m = ibcs_sip.target_count(w["ibcs"]["sample_frac"], (w["N"] + 15) // 16)
    cnt = L.cnt.cpu().numpy()
    assert abs(cnt.mean() - m) < 3.0, (cnt.mean(), m)


def test_weighted_attention_full_hunyuan_shape_sampled_blocks(hunyuan):
    """SIP-weighted attention at the full HunyuanVideo shape: about 743 sampled
    16-key units (93 tiles) per query block, log-weights up to ln(1/pi_min).
    The GPU output of the first, last and 6 seeded query blocks of heads 0,
    13 and 23 against the oracle over the same lists and weights."""
    api, session = _lib()
    w, q, k, v, L, qblocks = (hunyuan[x] for x in ("w", "q", "k", "v", "L", "qblocks"))
    o = torch.full_like(hunyuan["qd"], float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), hunyuan["qd"],
                            hunyuan["kd"], hunyuan["vd"], L.struct, o, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, api.sta_dev_status_string(int(st.item()))
    N = w["N"]
    nqb = (N + 127) // 128
    cnt = L.cnt.cpu().numpy()
    idx = L.idx.cpu().numpy()
    lw = L.logw.cpu().numpy()
    assert float(lw[cnt > 0].max()) > 1.0  # weights well away from 1 are exercised
    for h in (0, 13, 23):
        for qb in qblocks:
            r = h * nqb + qb
            units = idx[r, :cnt[r]].tolist()
            ref = block_sparse_rows(q[h], k[h], v[h], qb, units, 128, 16, lw[r, :cnt[r]])
            lo, hi = qb * 128, min(N, qb * 128 + 128)
            assert_close_attn(o[h, lo:hi].float().cpu().numpy(), ref, f"head {h} qb {qb}")


def test_sampled_attention_matches_oracle(cuda_ok):
    api, session = _lib()
    w = workload("ab_sampled", heads=3, F=6, H=20, W=32)   # N = 3840, 240 sub-blocks
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    L = _gpu_select(w, qd, kd)
    o = torch.full_like(qd, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), qd, kd, vd, L.struct, o,
                            dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    nqb = (w["N"] + 127) // 128
    rows = L.host_rows()
    lw = L.logw.cpu().numpy()
    oc = o.cpu()
    for h in range(3):
        for qb in range(nqb):
            r = h * nqb + qb
            ref = block_sparse_rows(q[h], k[h], v[h], qb, rows[r], 128, 16, lw[r, :len(rows[r])])
            lo, hi = qb * 128, min(w["N"], qb * 128 + 128)
            assert_close_attn(oc[h, lo:hi].float().numpy(), ref, f"head {h} qb {qb}")


def test_fraction_one_keeps_everything_unweighted(cuda_ok):
    api, session = _lib()
    w = workload("ab_sampled", heads=1, F=3, H=10, W=13)    # N = 390, ragged units
    w["ibcs"]["sample_frac"] = 1.0
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    L = _gpu_select(w, qd, kd)
    n_sub = (w["N"] + 15) // 16
    assert all(r == list(range(n_sub)) for r in L.host_rows())
    assert float(L.logw.abs().max()) <= 1e-6
    o = torch.empty_like(qd)
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), qd, kd, vd, L.struct, o)
    torch.cuda.synchronize()
    ref = np.concatenate([dense_rows(q[0], k[0], v[0], qb, 128) for qb in range(4)])
    assert_close_attn(o[0].float().cpu().numpy(), ref, "frac=1 vs dense")


@pytest.mark.parametrize("k,block_q", [(1, 128), (2, 128), (8, 128), (4, 64)])
def test_ibcs_centroid_counts_and_query_blocks(cuda_ok, k, block_q):
    """Other centroid counts and a 64-query block (ragged last block)."""
    w = workload("ab_sampled", heads=2, F=3, H=10, W=13, block_q=block_q)   # N = 390
    w["ibcs"]["k"] = k
    w["ibcs"]["sample_frac"] = 0.25
    q, k_, _ = make_qkv(w)
    L = _gpu_select(w, q.cuda(), k_.cuda())
    checked, skipped, near = _check_rows(w, L, q, k_, (0, 1), None)
    # k = 8 on the 6-query last block starts two centroids on the same query:
    # an exact tie (margin 0), so that row of each head is not compared
    assert checked >= 4 and skipped <= 2 and near <= 2
