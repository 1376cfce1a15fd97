"""GPU parity of the token-level TRA pipeline ("Token Radius Attention for
Efficient Video Generation", 2. Methodology: Insight I, Insight II, The TRA
Pipeline): the dense warm-up's per-query entropy, the entropy -> budget ->
disk -> token-voting block lists, and the sparse attention over them.

Entropies agree with the fp64 oracle to 2e-5 nats (fp32 accumulation of the
unrounded probabilities).  Lists are built on each side from its own
entropies and must match bit-exactly except key blocks whose decision rests
on a near-threshold (query, key) pair, which the oracle reports and the
tests count and bound.  Attention outputs are within the workload tolerance
(tests/_util.py)."""
import math

import numpy as np
import pytest
import torch

from oracle import tra_token
from oracle.pipeline import block_sparse_rows, dense_rows
from synthetic import make_qkv, workload
from tests._util import assert_close_attn

pytestmark = pytest.mark.gpu

ENT_TOL = 2e-5


def _api():
    from sparse_spatiotemporal_attention_video_b200 import api, session
    return api, session


def _warmup(w, qd, kd, vd):
    api, session = _api()
    o = torch.empty_like(qd)
    H = torch.full((w["heads"], w["N"]), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_dense_attn_entropy_fwd(session.problem(w), qd, kd, vd, 0.0, o, H, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, api.sta_dev_status_string(int(st.item()))
    return o, H


def _select(w, H):
    api, session = _api()
    L = session.Lists(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_build_blocks(session.problem(w), session.selector(w, entropy=H), None, None,
                         L.struct, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, api.sta_dev_status_string(int(st.item()))
    return L


def _check_lists(w, L, Href, heads, qblocks):
    """GPU rows against oracle rows built from the oracle entropies."""
    c = w["tra_token"]
    nqb = (w["N"] + w["block_q"] - 1) // w["block_q"]
    rows = L.host_rows()
    amb_total = checked = 0
    for h in heads:
        ref = tra_token.block_lists(Href[h], w["F"], w["H"], w["W"], w["block_q"], c["tau"],
                                    c["gamma"], c["vote"], qblocks)
        for qb, (ids, amb) in ref.items():
            got = rows[h * nqb + qb]
            assert got == sorted(got)
            diff = set(got) ^ set(ids.tolist())
            assert diff <= set(amb.tolist()), (h, qb, sorted(diff)[:8])
            amb_total += len(amb)
            checked += 1
    return checked, amb_total


@pytest.mark.parametrize("F,H,W,heads", [(4, 12, 16, 2), (5, 9, 14, 1)])
def test_small_grid_whole_pipeline(cuda_ok, F, H, W, heads):
    # N = 768 (6 full blocks) and N = 630 (a partial last block)
    w = workload("tra_token", F=F, H=H, W=W, heads=heads)
    w["tra_token"]["tau"] = 0.05  # keeps 78% and 56% of the blocks of these grids
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, Hd = _warmup(w, qd, kd, vd)
    d = w["d"]
    nqb = (w["N"] + 127) // 128
    Href = []
    for h in range(heads):
        ref = tra_token.query_entropy(q[h].float().numpy(), k[h].float().numpy(),
                                      1 / math.sqrt(d))
        assert np.abs(Hd[h].cpu().numpy() - ref).max() <= ENT_TOL
        Href.append(ref)
        for qb in range(nqb):
            lo, hi = qb * 128, min(w["N"], qb * 128 + 128)
            assert_close_attn(o[h, lo:hi].float().cpu().numpy(),
                              dense_rows(q[h], k[h], v[h], qb, 128), f"warm-up head {h} qb {qb}")
    L = _select(w, Hd)
    checked, amb = _check_lists(w, L, Href, range(heads), None)
    assert checked == heads * nqb and amb <= 2
    cnt = L.cnt.cpu().numpy()
    assert 0 < cnt.mean() < nqb  # neither empty nor dense
    # sparse attention over the lists
    api, session = _api()
    os_ = torch.full_like(qd, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), qd, kd, vd, L.struct,
                            os_, dev_status=st)
    torch.cuda.synchronize()
    rows = L.host_rows()
    for h in range(heads):
        for qb in range(nqb):
            r = rows[h * nqb + qb]
            lo, hi = qb * 128, min(w["N"], qb * 128 + 128)
            if not r:
                assert np.all(os_[h, lo:hi].float().cpu().numpy() == 0)
                continue
            ref = block_sparse_rows(q[h], k[h], v[h], qb, r, 128, 128)
            assert_close_attn(os_[h, lo:hi].float().cpu().numpy(), ref, f"head {h} qb {qb}")


def test_full_wan_shape_sampled_blocks(cuda_ok):
    w = workload("tra_token")
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    _, Hd = _warmup(w, qd, kd, vd)
    N, d = w["N"], w["d"]
    nqb = (N + 127) // 128
    qblocks = [0, 77, 150, nqb - 1]  # the last block is partial (120 tokens)
    heads = (0, 11)
    Href = {}
    for h in heads:
        ref = np.zeros(N)
        kh = k[h].float().numpy()
        for qb in qblocks:
            lo, hi = qb * 128, min(N, qb * 128 + 128)
            ref[lo:hi] = tra_token.query_entropy(q[h, lo:hi].float().numpy(), kh,
                                                 1 / math.sqrt(d))
            assert np.abs(Hd[h, lo:hi].cpu().numpy() - ref[lo:hi]).max() <= ENT_TOL
        Href[h] = ref
    L = _select(w, Hd)
    checked, amb = _check_lists(w, L, Href, heads, qblocks)
    # near-threshold key blocks: at most 1% of the block decisions checked
    # (10 of 2048 on these inputs)
    assert checked == len(heads) * len(qblocks) and amb <= 0.01 * checked * nqb
    # 9-19% of block pairs kept over the whole problem
    density = L.cnt.float().mean().item() / nqb
    assert 0.09 <= density <= 0.19, density
