"""The allocation-free attention entry point against the ordinary one.

sta_sparse_attn_fwd_noalloc exists for callers that cannot allocate device
memory (a plugin given only its input and output buffers, or a pipeline that
bans cudaMalloc after start-up because it can synchronise the device).  For
fp32 inputs it stages the bf16 copies in a fixed array inside the library
instead of a caller workspace.  These tests call both entry points through
the C ABI on the same inputs and lists, twice in a row with different inputs
(the second call must not see the first call's leftovers), at the largest
size the fixed array holds, and check that an fp32 problem larger than the
fixed array is refused before any work.

The file name sorts last so that a stop-at-first-failure run has executed
every other test before this one.
"""
import ctypes

import pytest
import torch

from synthetic import make_qkv, workload

pytestmark = pytest.mark.gpu


def _lists_for(w):
    from sparse_spatiotemporal_attention_video_b200 import api, session
    L = session.Lists(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_build_blocks(session.problem(w), session.selector(w), None, None, L.struct,
                         dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return L


def _with_workspace(w, q, k, v, L):
    from sparse_spatiotemporal_attention_video_b200 import api, session
    prob = session.problem(w)
    ws = torch.empty(max(1, api.sta_attn_workspace(prob)), dtype=torch.uint8, device="cuda")
    o = torch.full(q.shape, float("nan"), dtype=q.dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.sta_sparse_attn_fwd(prob, session.attn_params(w), q, k, v, L.struct, o, workspace=ws,
                            dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return o


def _no_alloc(w, q, k, v, L):
    from sparse_spatiotemporal_attention_video_b200 import _lib, session
    lib = _lib.load()
    o = torch.full(q.shape, float("nan"), dtype=q.dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    code = lib.sta_sparse_attn_fwd_noalloc(
        ctypes.byref(session.problem(w)), ctypes.byref(session.attn_params(w)), q.data_ptr(),
        k.data_ptr(), v.data_ptr(), ctypes.byref(L.struct), o.data_ptr(), st.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert code == _lib.STA_OK, code
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return o


@pytest.mark.parametrize("name", ["tiny_radial", "tiny_radial_b16"])
def test_no_alloc_matches_workspace_entry_on_two_calls(cuda_ok, name):
    w = workload(name)
    assert w["dtype"] == "f32"  # the case that needs scratch
    L = _lists_for(w)
    for seed in (11, 12):
        q, k, v = (x.cuda() for x in make_qkv(dict(w, seed=seed)))
        ref = _with_workspace(w, q, k, v, L)
        got = _no_alloc(w, q, k, v, L)
        # both entries run the same conversion and attention kernels on the
        # same staged bf16 bytes: the outputs are identical, not just close
        assert torch.equal(got, ref), f"{name} seed {seed}"


def test_no_alloc_bf16_needs_no_scratch(cuda_ok):
    w = workload("wan_radial", heads=2, F=3, H=10, W=13)
    L = _lists_for(w)
    q, k, v = (x.cuda() for x in make_qkv(w))
    ref = _with_workspace(w, q, k, v, L)
    got = _no_alloc(w, q, k, v, L)
    assert torch.equal(got, ref)


def test_no_alloc_at_the_size_limit(cuda_ok):
    """1 head x 16,384 tokens x 128 = 2,097,152 elements per tensor: the three
    bf16 copies fill the 12 MiB array exactly, and the call must succeed."""
    w = workload("tiny_radial", F=1, H=128, W=128, d=128, block_q=128, kv_unit=128)
    assert w["heads"] * w["N"] * w["d"] == 2_097_152
    L = _lists_for(w)
    for seed in (21, 22):
        q, k, v = (x.cuda() for x in make_qkv(dict(w, seed=seed)))
        ref = _with_workspace(w, q, k, v, L)
        got = _no_alloc(w, q, k, v, L)
        assert torch.equal(got, ref), f"seed {seed}"


def test_no_alloc_refuses_problems_beyond_the_fixed_array(cuda_ok):
    from sparse_spatiotemporal_attention_video_b200 import _lib, session
    lib = _lib.load()
    # 1 head x 16,400 tokens x 128 = 2,099,200 elements per tensor: above the
    # 2,097,152 the 12 MiB array holds for three bf16 copies.
    w = workload("tiny_radial", F=1, H=100, W=164, d=128, block_q=128, kv_unit=128)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    lists = _lib.BlockLists()     # valid-looking lists: only the size is wrong
    lists.idx, lists.cnt, lists.cap = dummy.data_ptr(), dummy.data_ptr(), 1
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (ctypes.byref(session.problem(w)), ctypes.byref(session.attn_params(w)),
            dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), ctypes.byref(lists),
            dummy.data_ptr(), st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    code = lib.sta_sparse_attn_fwd_noalloc(*args)
    assert code == _lib.STA_ERR_WORKSPACE
    # argument errors are reported before the size check, as by the ordinary
    # entry point: a null output pointer is STA_ERR_ARG
    bad = list(args)
    bad[6] = None
    assert lib.sta_sparse_attn_fwd_noalloc(*bad) == _lib.STA_ERR_ARG
    torch.cuda.synchronize()
    assert int(st.item()) == 0
