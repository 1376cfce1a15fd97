"""GPU parity of the tile-major token order ("Token Radius Attention for
Efficient Video Generation", 2. Methodology, The TRA Pipeline, Efficient
Execution: tokens reordered tile by tile so that a query's spatial neighbours
are contiguous).

- sta_permute_tokens moves rows into the oracle's tile-major order
  (oracle/tile_major.py) and back, bit-exactly, for ragged tiles, both element
  types and both head dimensions; t_h = 1, t_w = W is the identity.
- The token-level selector in that order (layout_tile_h/w) gives the oracle's
  lists over blocks of tile-major positions (tra_token.block_lists with
  perm), bit-exactly except key blocks decided by near-threshold pairs.
- Attention over the permuted q, k, v with those lists, permuted back, equals
  the oracle within the workload tolerance (tests/_util.py).
"""
import math

import numpy as np
import pytest
import torch

from oracle import tile_major, tra_token
from oracle.pipeline import block_sparse_rows
from synthetic import make_qkv, workload
from tests._util import assert_close_attn

pytestmark = pytest.mark.gpu

ENT_TOL = 2e-5


def _api():
    from sparse_spatiotemporal_attention_video_b200 import api, session
    return api, session


def _permute(w, x, th, tw, inverse):
    api, session = _api()
    out = torch.empty_like(x)
    api.sta_permute_tokens(session.problem(w), th, tw, inverse, x, out)
    return out


@pytest.mark.parametrize("F,H,W,th,tw", [(2, 8, 16, 3, 5), (3, 10, 13, 4, 4), (2, 6, 20, 1, 20),
                                         (1, 16, 32, 16, 8)])
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "bf16"), (128, "f32"), (64, "f32")])
def test_permutation_matches_oracle_order(cuda_ok, F, H, W, th, tw, d, dtype):
    w = workload("tra_token", heads=2, F=F, H=H, W=W, d=d, dtype=dtype)
    q, _, _ = make_qkv(w)
    qd = q.cuda()
    perm = torch.from_numpy(tile_major.order(F, H, W, th, tw))
    tiled = _permute(w, qd, th, tw, 0)
    torch.cuda.synchronize()
    assert torch.equal(tiled.cpu(), q[:, perm])
    back = _permute(w, tiled, th, tw, 1)
    torch.cuda.synchronize()
    assert torch.equal(back.cpu(), q)
    if th == 1 and tw == W:
        assert torch.equal(tiled.cpu(), q)  # raster order is the identity


def _pipeline(w, q, k, v, th, tw):
    """GPU: permute q, k, v; dense warm-up with per-query entropy in the
    tile-major order; token-level lists in that order.  Returns the permuted
    device tensors, the entropies (by position) and the lists."""
    api, session = _api()
    qt, kt, vt = (_permute(w, x.cuda(), th, tw, 0) for x in (q, k, v))
    o = torch.empty_like(qt)
    H = torch.full((w["heads"], w["N"]), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_dense_attn_entropy_fwd(session.problem(w), qt, kt, vt, 0.0, o, H, dev_status=st)
    L = session.Lists(w)
    api.sta_build_blocks(session.problem(w), session.selector(w, entropy=H), None, None,
                         L.struct, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, api.sta_dev_status_string(int(st.item()))
    return qt, kt, vt, H, L


def _check_lists(w, L, Href, perm, heads, qblocks):
    c = w["tra_token"]
    nqb = (w["N"] + w["block_q"] - 1) // w["block_q"]
    rows = L.host_rows()
    amb_total = checked = 0
    for h in heads:
        ref = tra_token.block_lists(Href[h], w["F"], w["H"], w["W"], w["block_q"], c["tau"],
                                    c["gamma"], c["vote"], qblocks, perm=perm)
        for qb, (ids, amb) in ref.items():
            got = rows[h * nqb + qb]
            assert got == sorted(got)
            diff = set(got) ^ set(ids.tolist())
            assert diff <= set(amb.tolist()), (h, qb, sorted(diff)[:8])
            amb_total += len(amb)
            checked += 1
    return checked, amb_total


@pytest.mark.parametrize("F,H,W,th,tw", [(3, 16, 32, 8, 16), (2, 10, 24, 4, 16),
                                         (3, 16, 32, 16, 8)])
def test_tile_layout_lists_and_attention_match_oracle(cuda_ok, F, H, W, th, tw):
    # N = 1,536 / 480: several blocks, ragged tiles in the second grid
    w = workload("tra_token", heads=2, F=F, H=H, W=W, layout=(th, tw))
    w["tra_token"]["tau"] = 0.05
    q, k, v = make_qkv(w)
    perm = tile_major.order(F, H, W, th, tw)
    qt, kt, vt, Hd, L = _pipeline(w, q, k, v, th, tw)
    d, N = w["d"], w["N"]
    nqb = (N + 127) // 128
    Href = []
    for h in range(2):
        ref = tra_token.query_entropy(q[h].float().numpy(), k[h].float().numpy(),
                                      1 / math.sqrt(d))  # by raster token
        assert np.abs(Hd[h].cpu().numpy() - ref[perm]).max() <= ENT_TOL
        Href.append(ref)
    checked, amb = _check_lists(w, L, Href, perm, range(2), None)
    assert checked == 2 * nqb and amb <= 2
    cnt = L.cnt.cpu().numpy()
    assert 0 < cnt.mean() < nqb
    # attention in the tile-major order, output permuted back
    api, session = _api()
    ot = torch.full_like(qt, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), qt, kt, vt, L.struct,
                            ot, dev_status=st)
    o = _permute(w, ot, th, tw, 1)
    torch.cuda.synchronize()
    rows = L.host_rows()
    oc = o.cpu()
    for h in range(2):
        qp, kp, vp = (tile_major.to_layout(x[h].float().numpy(), perm) for x in (q, k, v))
        ref_t = np.zeros((N, d))
        for qb in range(nqb):
            lo, hi = qb * 128, min(N, qb * 128 + 128)
            r = rows[h * nqb + qb]
            if r:
                ref_t[lo:hi] = block_sparse_rows(qp, kp, vp, qb, r, 128, 128)
        got_t = tile_major.to_layout(oc[h].float().numpy(), perm)
        assert_close_attn(got_t, ref_t, f"head {h}")
        # the permuted-back output is the oracle's rows in raster order
        assert_close_attn(oc[h].float().numpy(), tile_major.from_layout(ref_t, perm),
                          f"head {h} raster")


def test_tiled_workload_full_shape_sampled_blocks(cuda_ok):
    w = workload("tra_token_tiled")
    th, tw = w["layout"]
    q, k, v = make_qkv(w)
    perm = tile_major.order(w["F"], w["H"], w["W"], th, tw)
    _, _, _, Hd, L = _pipeline(w, q, k, v, th, tw)
    N, d = w["N"], w["d"]
    nqb = (N + 127) // 128
    qblocks = [0, 131, 260, nqb - 1]
    heads = (0, 11)
    Href = {}
    for h in heads:
        ref = np.zeros(N)
        kh = k[h].float().numpy()
        for qb in qblocks:
            toks = perm[qb * 128:min(N, qb * 128 + 128)]
            ref[toks] = tra_token.query_entropy(q[h, toks].float().numpy(), kh,
                                                1 / math.sqrt(d))
            assert np.abs(Hd[h, qb * 128:qb * 128 + len(toks)].cpu().numpy()
                          - ref[toks]).max() <= ENT_TOL
        Href[h] = ref
    checked, amb = _check_lists(w, L, Href, perm, heads, qblocks)
    assert checked == len(heads) * len(qblocks) and amb <= 0.01 * checked * nqb
    density = L.cnt.float().mean().item() / nqb
    assert 0.09 <= density <= 0.19, density
