"""CPU checks of the C-ABI library: it loads without a GPU, exports every
function include/sta.h declares, and rejects bad arguments on the host."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    txt = open(os.path.join(ROOT, "include", "sta.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"\b(sta_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from sparse_spatiotemporal_attention_video_b200 import _lib
    return _lib.load()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["sta_build_blocks", "sta_sparse_attn_fwd", "sta_dense_attn_fwd"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n


def test_binding_signatures_cover_the_header():
    from sparse_spatiotemporal_attention_video_b200 import _lib
    assert set(_declared_functions()) <= set(_lib.SIGNATURES)


def test_version_and_strings(lib):
    from sparse_spatiotemporal_attention_video_b200 import api
    assert api.sta_version() >= 100
    assert api.sta_status_string(-2).startswith("unsupported")
    assert api.sta_dev_status_string(0) == "ok"
    assert "timeout" in api.sta_dev_status_string(1)


def test_host_argument_checks(lib):
    from sparse_spatiotemporal_attention_video_b200._lib import (
        STA_ERR_ARG, STA_ERR_UNSUPPORTED, AttnParams, BlockLists, Problem, SelectorParams)
    sel = SelectorParams()
    sel.block_q = sel.kv_unit = 128
    lists = BlockLists()
    bad = Problem(0, 4, 8, 8, 64, 0)
    assert lib.sta_build_blocks(ctypes.byref(bad), ctypes.byref(sel), None, None,
                                ctypes.byref(lists), None, 0, None, None) == STA_ERR_ARG
    odd_d = Problem(1, 4, 8, 8, 96, 0)
    assert lib.sta_dense_attn_fwd(ctypes.byref(odd_d), 1, 1, 1, 0.0, 1, None, 0, None,
                                  None) == STA_ERR_UNSUPPORTED
    good = Problem(1, 4, 8, 8, 64, 0)
    # missing list buffers
    assert lib.sta_build_blocks(ctypes.byref(good), ctypes.byref(sel), None, None,
                                ctypes.byref(lists), None, 0, None, None) == STA_ERR_ARG
    prm = AttnParams()
    prm.block_q, prm.kv_unit = 128, 48          # not a supported unit
    assert lib.sta_sparse_attn_fwd(ctypes.byref(good), ctypes.byref(prm), 1, 1, 1,
                                   ctypes.byref(lists), 1, None, 0, None,
                                   None) == STA_ERR_UNSUPPORTED
    assert lib.sta_build_blocks_rows(ctypes.byref(good), ctypes.byref(sel)) == 2
    assert lib.sta_attn_workspace(ctypes.byref(Problem(2, 4, 8, 8, 64, 1))) == 3 * 2 * 256 * 64 * 2


def test_selftest_argument_checks(lib):
    from sparse_spatiotemporal_attention_video_b200._lib import STA_ERR_ARG
    assert lib.sta_selftest_bounded_wait(0, 1, 1, None) == STA_ERR_ARG
    assert lib.sta_selftest_bounded_wait(10**10, 1, 1, None) == STA_ERR_ARG
    assert lib.sta_selftest_bounded_wait(1000, None, 1, None) == STA_ERR_ARG


def test_next_selector_argument_checks(lib):
    """Host checks of the token-level and radial-prior selectors and of the
    entropy-writing dense entry point; every case returns before a launch."""
    from sparse_spatiotemporal_attention_video_b200._lib import (
        STA_ERR_ARG, STA_ERR_UNSUPPORTED, STA_ERR_WORKSPACE, STA_SEL_DYNRAD,
        STA_SEL_TRA_TOKEN, BlockLists, Problem, SelectorParams)
    good = Problem(2, 4, 8, 8, 64, 0)  # 2 heads, 256 tokens, two 128-blocks
    lists = BlockLists()
    lists.idx, lists.cnt, lists.cap = 256, 512, 4  # never dereferenced on these paths
    fake = ctypes.c_void_p(4096)

    def build(sel, prob=good, q=fake, k=fake):
        return lib.sta_build_blocks(ctypes.byref(prob), ctypes.byref(sel), q, k,
                                    ctypes.byref(lists), None, 0, None, None)

    tra = SelectorParams()
    tra.kind, tra.block_q, tra.kv_unit = STA_SEL_TRA_TOKEN, 128, 128
    tra.tra_tau, tra.tra_gamma, tra.tra_vote = 0.07, 0.25, 1
    assert build(tra) == STA_ERR_ARG                       # no entropy buffer
    tra.tra_entropy = 8192
    for field, bad in (("tra_tau", 0.0), ("tra_tau", float("nan")), ("tra_gamma", -0.5),
                       ("tra_vote", 0)):
        saved = getattr(tra, field)
        setattr(tra, field, bad)
        assert build(tra) == STA_ERR_ARG, field
        setattr(tra, field, saved)
    tra.kv_unit = 64
    assert build(tra) == STA_ERR_UNSUPPORTED               # token lists are block_q wide
    tra.kv_unit = 128
    assert build(tra, Problem(1, 2000, 4, 4, 64, 0)) == STA_ERR_UNSUPPORTED  # > frame limit
    assert lib.sta_build_blocks_rows(ctypes.byref(good), ctypes.byref(tra)) == 2 * 2
    assert lib.sta_build_blocks_workspace(ctypes.byref(good), ctypes.byref(tra)) == 0
    # tile-major token order: both tile sides or neither, within the grid
    for th, tw in ((4, 0), (0, 4), (-1, 4), (9, 4), (4, 9)):
        tra.layout_tile_h, tra.layout_tile_w = th, tw
        assert build(tra) == STA_ERR_ARG, (th, tw)
    tra.layout_tile_h = tra.layout_tile_w = 0

    dyn = SelectorParams()
    dyn.kind, dyn.block_q, dyn.kv_unit = STA_SEL_DYNRAD, 128, 128
    dyn.radial_w0, dyn.radial_w_off, dyn.radial_full_df = 8, 1, 1
    dyn.dyn_mode, dyn.dyn_ratio, dyn.dyn_threshold = 0, 0.35, 0.35
    assert build(dyn, q=None) == STA_ERR_ARG               # needs q and k
    assert build(dyn, Problem(2, 4, 8, 8, 64, 1)) == STA_ERR_UNSUPPORTED  # bf16 inputs only
    for mode, ratio, thr in ((2, 0.35, 0.35), (0, 0.0, 0.35), (0, 1.5, 0.35),
                             (1, 0.35, 0.0), (1, 0.35, float("nan"))):
        dyn.dyn_mode, dyn.dyn_ratio, dyn.dyn_threshold = mode, ratio, thr
        assert build(dyn) == STA_ERR_ARG, (mode, ratio, thr)
    dyn.dyn_mode, dyn.dyn_ratio = 0, 1.0
    dyn.kv_unit = 64
    assert build(dyn) == STA_ERR_UNSUPPORTED
    dyn.kv_unit = 128
    # candidate limit: 1025 blocks of 128 tokens exceed the per-CTA candidate buffer
    assert build(dyn, Problem(1, 1025, 8, 16, 64, 0)) == STA_ERR_UNSUPPORTED
    ws = lib.sta_build_blocks_workspace(ctypes.byref(good), ctypes.byref(dyn))
    # block means of q and k (fp32) and the prior lists fit in the workspace
    assert ws >= 2 * 2 * 2 * 64 * 4 + 2 * 2 * 4 + 2 * 4
    assert build(dyn) == STA_ERR_WORKSPACE                 # no workspace given
    assert lib.sta_build_blocks_rows(ctypes.byref(good), ctypes.byref(dyn)) == 2 * 2

    assert lib.sta_dense_attn_entropy_fwd(ctypes.byref(good), fake, fake, fake, 0.0, fake,
                                          None, None, 0, None, None) == STA_ERR_ARG
    assert lib.sta_dense_attn_entropy_fwd(ctypes.byref(Problem(1, 4, 8, 8, 96, 0)), fake, fake,
                                          fake, 0.0, fake, fake, None, 0, None,
                                          None) == STA_ERR_UNSUPPORTED


def test_binding_rejects_views_and_host_tensors():
    import pytest
    import torch
    from sparse_spatiotemporal_attention_video_b200 import api
    with pytest.raises(ValueError, match="contiguous"):
        api._ptr(torch.zeros(4, 8).t())
    with pytest.raises(ValueError, match="device"):
        api._ptr(torch.zeros(4, 8))
    with pytest.raises(TypeError):
        api._ptr([1, 2])
    assert api._ptr(None) is None and api._ptr(4096) == 4096


def test_package_exports_every_selector_kind(lib):
    import sparse_spatiotemporal_attention_video_b200 as pkg
    from sparse_spatiotemporal_attention_video_b200 import _lib
    kinds = [n for n in dir(_lib) if n.startswith("STA_SEL_")]
    assert len(kinds) == 6
    for n in kinds:
        assert getattr(pkg, n) == getattr(_lib, n), n


def test_permute_tokens_argument_checks(lib):
    """sta_permute_tokens rejects null and overlapping buffers and tiles
    outside the grid before any launch."""
    from sparse_spatiotemporal_attention_video_b200._lib import (STA_ERR_ARG,
                                                                 STA_ERR_UNSUPPORTED, Problem)
    good = Problem(2, 4, 8, 8, 64, 0)        # bf16 rows of 128 bytes, 2 x 256 rows: 64 KiB
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 24)

    def perm(th, tw, x=a, y=b, prob=good):
        return lib.sta_permute_tokens(ctypes.byref(prob), th, tw, 0, x, y, None)

    assert perm(4, 4, None, b) == STA_ERR_ARG
    assert perm(4, 4, a, None) == STA_ERR_ARG
    for th, tw in ((0, 4), (4, 0), (9, 4), (4, 9), (-2, 2)):
        assert perm(th, tw) == STA_ERR_ARG, (th, tw)
    assert perm(4, 4, a, ctypes.c_void_p((1 << 20) + 4096)) == STA_ERR_ARG  # overlap
    assert perm(4, 4, a, ctypes.c_void_p((1 << 24) + 8)) == STA_ERR_ARG    # not 16-byte aligned
    assert perm(4, 4, prob=Problem(2, 4, 8, 8, 96, 0)) == STA_ERR_UNSUPPORTED
