"""GPU parity of difficulty routing (dense path for the hardest tokens, a
local 3D window for the rest) against the fp64 oracle: the routed set is
bit-exact, the local unit lists cover exactly the units that hold a window
key, and the attention of both paths matches the oracle."""
import numpy as np
import pytest
import torch

from oracle import routed
from oracle.pipeline import routed_rows
from synthetic import make_difficulty, make_qkv, workload
from tests._util import assert_close_attn

pytestmark = pytest.mark.gpu


def _lib():
    from sparse_spatiotemporal_attention_video_b200 import api, session
    return api, session


def _gpu_route(w, dif):
    api, session = _lib()
    L = session.Lists(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dd = torch.from_numpy(dif).cuda()
    api.sta_build_blocks(session.problem(w), session.selector(w, dd), None, None, L.struct,
                         dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, api.sta_dev_status_string(int(st.item()))
    return L


def _units_with_window_keys(w):
    """Brute force: units holding a key in the window of some query of the block."""
    F, H, W, B, U = w["F"], w["H"], w["W"], w["block_q"], w["kv_unit"]
    c = w["routed"]
    N = F * H * W
    out = []
    for qb in range((N + B - 1) // B):
        units = set()
        for t in range(qb * B, min(N, qb * B + B)):
            keys = routed.window_keys(t, F, H, W, c["win_f"], c["win_h"], c["win_w"])
            units.update((keys // U).tolist())
        out.append(sorted(units))
    return out


@pytest.mark.parametrize("shape", [(31, 44, 80), (3, 10, 13), (4, 7, 40)])
def test_routed_set_bit_exact(cuda_ok, shape):
    F, H, W = shape
    w = workload("heta_routed", F=F, H=H, W=W)
    dif = make_difficulty(w)
    L = _gpu_route(w, dif)
    ref = routed.route(dif, w["routed"]["dense_frac"])
    n = L.struct.n_routed
    assert n == len(ref)
    assert L.routed_ids[:n].cpu().numpy().tolist() == ref.tolist()
    flag = np.zeros(w["N"], np.uint8)
    flag[ref] = 1
    assert np.array_equal(L.routed_flag.cpu().numpy(), flag)


def test_routed_ties_go_to_lower_index(cuda_ok):
    w = workload("heta_routed", F=2, H=8, W=16)      # N = 256, 52 routed
    dif = np.full(w["N"], 0.25, np.float32)
    dif[200:] = 0.5                                   # 56 tokens above the tie level
    dif[10] = -0.0
    dif[11] = 0.0
    L = _gpu_route(w, dif)
    ref = routed.route(dif, w["routed"]["dense_frac"])
    n = L.struct.n_routed
    assert L.routed_ids[:n].cpu().numpy().tolist() == ref.tolist()
    dif[:] = 0.3                                      # all equal: the lowest ids win
    L = _gpu_route(w, dif)
    assert L.routed_ids[:n].cpu().numpy().tolist() == list(range(n))


@pytest.mark.parametrize("shape,B,U", [((3, 10, 13), 128, 16), ((4, 12, 20), 64, 32),
                                       ((2, 20, 9), 128, 16)])
def test_local_lists_equal_window_units(cuda_ok, shape, B, U):
    F, H, W = shape
    w = workload("heta_routed", F=F, H=H, W=W, block_q=B, kv_unit=U)
    L = _gpu_route(w, make_difficulty(w))
    assert L.host_rows() == _units_with_window_keys(w)


@pytest.mark.parametrize("shape", [(3, 10, 13), (4, 12, 20)])
def test_routed_attention_whole_small_grid(cuda_ok, shape):
    api, session = _lib()
    F, H, W = shape
    w = workload("heta_routed", heads=2, F=F, H=H, W=W)
    q, k, v = make_qkv(w)
    dif = make_difficulty(w)
    L = _gpu_route(w, dif)
    o = torch.full_like(q, float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), q.cuda(), k.cuda(),
                            v.cuda(), L.struct, o, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    flag = L.routed_flag.cpu().numpy().astype(bool)
    c = w["routed"]
    oc = o.cpu()
    for h in range(2):
        ref = routed_rows(q[h], k[h], v[h], np.arange(w["N"]), flag, F, H, W, c["win_f"],
                          c["win_h"], c["win_w"])
        assert_close_attn(oc[h].float().numpy(), ref, f"head {h}")


def test_routed_attention_sampled_tokens_wan22_shape(cuda_ok):
    api, session = _lib()
    w = workload("heta_routed")
    q, k, v = make_qkv(w)
    dif = make_difficulty(w)
    L = _gpu_route(w, dif)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.full_like(qd, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(session.problem(w), session.attn_params(w), qd, kd, vd, L.struct, o,
                            dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    flag = L.routed_flag.cpu().numpy().astype(bool)
    rng = np.random.default_rng(11)
    ids = L.routed_ids[:L.struct.n_routed].cpu().numpy()
    local = np.nonzero(~flag)[0]
    toks = np.concatenate([ids[[0, -1]], rng.choice(ids, 30, replace=False),
                           local[[0, -1]], rng.choice(local, 30, replace=False)])
    c = w["routed"]
    oc = o.cpu()
    for h in (0, 23):
        ref = routed_rows(q[h], k[h], v[h], toks, flag, w["F"], w["H"], w["W"], c["win_f"],
                          c["win_h"], c["win_w"])
        assert_close_attn(oc[h, toks].float().numpy(), ref, f"head {h}")
