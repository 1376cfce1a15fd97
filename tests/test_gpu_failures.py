"""Failure detection without a GPU fault: a bounded wait that runs out
reports STA_DEV_TIMEOUT and leaves the context usable; list rows longer than
their capacity are truncated, flagged and their true length reported; an
out-of-range list entry or routed token id is skipped and flagged."""
import numpy as np
import pytest
import torch

from oracle import radial
from oracle.pipeline import block_sparse_rows
from synthetic import make_qkv, workload
from tests._util import assert_close_attn

pytestmark = pytest.mark.gpu


def _mods():
    from sparse_spatiotemporal_attention_video_b200 import _lib, api, session
    return _lib, api, session


def test_bounded_wait_times_out_and_context_survives(cuda_ok):
    _lib, api, session = _mods()
    lib = _lib.load()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    code = lib.sta_selftest_bounded_wait(50_000_000, st.data_ptr(), waited.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    assert code == _lib.STA_OK
    torch.cuda.synchronize()
    assert int(waited.item()) == 0
    assert int(st.item()) & _lib.STA_DEV_TIMEOUT
    # the context is still usable: a normal dense call gives the right result
    w = workload("wan_radial", heads=1, F=2, H=8, W=16)
    q, k, v = make_qkv(w)
    o = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_dense_attn_fwd(session.problem(w), q.cuda(), k.cuda(), v.cuda(), 0.0, o,
                           dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    ref = np.concatenate([block_sparse_rows(q[0], k[0], v[0], b, list(range(2)), 128, 128)
                          for b in range(2)])
    assert_close_attn(o[0].float().cpu().numpy(), ref, "dense after timeout")


def test_capacity_overflow_truncates_and_reports(cuda_ok):
    _lib, api, session = _mods()
    w = workload("wan_radial")
    ref = radial.block_lists(w["F"], w["H"], w["W"], w["block_q"], w["radial"])
    need = max(len(r) for r in ref)
    cap = need // 3
    L = session.Lists(w, cap=cap)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_build_blocks(session.problem(w), session.selector(w), None, None, L.struct,
                         dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & _lib.STA_DEV_CAPACITY
    assert int(L.required_cap.item()) == need
    got = L.host_rows()
    for qb, r in enumerate(ref):
        assert got[qb] == list(r)[:cap]


def test_out_of_range_entry_is_skipped_and_flagged(cuda_ok):
    _lib, api, session = _mods()
    from sparse_spatiotemporal_attention_video_b200._lib import AttnParams, BlockLists
    w = workload("wan_radial", heads=1, F=3, H=10, W=13, kv_unit=32)   # N = 390
    q, k, v = make_qkv(w)
    n_units = (w["N"] + 31) // 32
    idx = np.array([[0, 3, n_units + 5, 7], [1, 2, 4, 9], [5, -1, 6, 10], [11, 12, 0, 0]],
                   np.int32)
    cnt = np.array([4, 4, 4, 2], np.int32)
    di, dc = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    L = BlockLists()
    L.idx, L.cnt, L.cap, L.head_shared = di.data_ptr(), dc.data_ptr(), 4, 0
    prm = AttnParams()
    prm.mode, prm.block_q, prm.kv_unit, prm.scale = 0, 128, 32, 0.0
    o = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(session.problem(w), prm, q.cuda(), k.cuda(), v.cuda(), L, o,
                            dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & _lib.STA_DEV_BAD_INDEX
    oc = o.cpu()
    for qb in range(4):
        units = [u for u in idx[qb, :cnt[qb]].tolist() if 0 <= u < n_units]
        lo, hi = qb * 128, min(w["N"], qb * 128 + 128)
        ref = block_sparse_rows(q[0], k[0], v[0], qb, units, 128, 32)
        assert_close_attn(oc[0, lo:hi].float().numpy(), ref, f"qb {qb}")


def test_out_of_range_routed_id_is_skipped_and_flagged(cuda_ok):
    """A routed id outside [0, N) in caller-written lists is neither read nor
    written: its row is skipped, STA_DEV_BAD_INDEX is raised, and every other
    row still equals the oracle."""
    _lib, api, session = _mods()
    from oracle.pipeline import routed_rows
    from synthetic import make_difficulty
    w = workload("heta_routed", heads=1, F=3, H=10, W=13)    # N = 390, 78 routed
    q, k, v = make_qkv(w)
    dif = make_difficulty(w)
    L = session.Lists(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_build_blocks(session.problem(w), session.selector(w, torch.from_numpy(dif).cuda()),
                         None, None, L.struct, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    n = L.struct.n_routed
    ids = L.routed_ids[:n].cpu().numpy().copy()
    flag = L.routed_flag.cpu().numpy().astype(bool)
    lost = ids[[3, n - 1]].copy()                 # these rows are skipped
    L.routed_ids[3] = w["N"] + 7
    L.routed_ids[n - 1] = -3
    o = torch.full_like(q, float("nan"), device="cuda")
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), q.cuda(), k.cuda(),
                            v.cuda(), L.struct, o, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & _lib.STA_DEV_BAD_INDEX
    oc = o[0].cpu().float().numpy()
    assert np.isnan(oc[lost]).all()               # skipped rows stay untouched
    keep = np.setdiff1d(np.arange(w["N"]), lost)
    c = w["routed"]
    ref = routed_rows(q[0], k[0], v[0], keep, flag, w["F"], w["H"], w["W"], c["win_f"],
                      c["win_h"], c["win_w"])
    assert_close_attn(oc[keep], ref, "rows with valid ids")


def test_misaligned_workspace_is_rejected(cuda_ok):
    """The selector workspace must start on a 256-byte boundary (its segments
    feed TMA descriptors and 16-byte stores); another start is an argument
    error reported before any launch."""
    _lib, api, session = _mods()
    w = workload("ab_sampled", heads=1, F=2, H=8, W=16)
    q, k, _ = make_qkv(w)
    need = api.sta_build_blocks_workspace(session.problem(w), session.selector(w))
    ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    L = session.Lists(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(_lib.StaError) as e:
        api.sta_build_blocks(session.problem(w), session.selector(w), q.cuda(), k.cuda(),
                             L.struct, workspace=ws.data_ptr() + 16, workspace_bytes=need,
                             dev_status=st)
    assert e.value.code == _lib.STA_ERR_WORKSPACE
    # the aligned start of the same buffer works
    api.sta_build_blocks(session.problem(w), session.selector(w), q.cuda(), k.cuda(), L.struct,
                         workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
