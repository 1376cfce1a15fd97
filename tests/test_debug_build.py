"""CPU checks of the debug build (libsta_debug.so, build.py --debug): it
loads without a GPU, exports every call include/sta.h declares, reports
itself as the debug build, and both libraries refuse the index-check
self-test's bad arguments on the host.  libsta.so refuses the self-test
itself (it has no checks to exercise)."""
import ctypes
import importlib.util
import os

import pytest

from tests.test_lib_abi import _declared_functions

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_spatiotemporal_attention_video_b200")


def debug_lib_path():
    """Path of libsta_debug.so, built from the current sources if missing."""
    path = os.path.join(PKG, "libsta_debug.so")
    if not os.path.exists(path):
        spec = importlib.util.spec_from_file_location("_sta_build", os.path.join(PKG, "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build(debug=True)
    return path


def load_with_signatures(path):
    from sparse_spatiotemporal_attention_video_b200 import _lib
    lib = ctypes.CDLL(path)
    for name, (res, args) in _lib.SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


@pytest.fixture(scope="module")
def dbg():
    return load_with_signatures(debug_lib_path())


@pytest.fixture(scope="module")
def rel():
    return load_with_signatures(os.path.join(PKG, "libsta.so"))


def test_debug_library_exports_every_declared_symbol(dbg):
    for n in _declared_functions():
        assert hasattr(dbg, n), n
    assert dbg.sta_version() >= 100


def test_debug_flag(dbg, rel):
    assert dbg.sta_debug_build() == 1
    assert rel.sta_debug_build() == 0


def test_index_check_selftest_host_refusals(dbg, rel):
    from sparse_spatiotemporal_attention_video_b200._lib import STA_ERR_ARG, STA_ERR_UNSUPPORTED
    for lib in (dbg, rel):
        assert lib.sta_selftest_index_check(None, 4, 0, 1, None) == STA_ERR_ARG
        assert lib.sta_selftest_index_check(1, 4, 0, None, None) == STA_ERR_ARG
        assert lib.sta_selftest_index_check(1, 0, 0, 1, None) == STA_ERR_ARG
    # the release library launches nothing (the dummy pointers are never used)
    assert rel.sta_selftest_index_check(1, 4, 7, 1, None) == STA_ERR_UNSUPPORTED


def test_status_string_names_the_debug_bit(dbg):
    from sparse_spatiotemporal_attention_video_b200._lib import STA_DEV_DEBUG
    assert b"debug" in dbg.sta_dev_status_string(STA_DEV_DEBUG)
    assert b"debug" in dbg.sta_dev_status_string(STA_DEV_DEBUG | 0x1)
