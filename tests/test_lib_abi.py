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
