"""The debug build on the GPU (libsta_debug.so: every kernel checks the
list entries, token indices and TMEM columns it uses, raises STA_DEV_DEBUG
and skips the access on a failed check).

- Its index check, driven by the self-test kernel: an in-range index is
  stored, an out-of-range one raises STA_DEV_DEBUG and stores nothing.  (The
  buffer is a 64-element torch allocation, whose 512-byte block also holds
  element 64, so even a broken check could not fault.)
- The parity tests of every selector and of the attention, run against the
  debug build (STA_LIB=debug in a child process): every device status must
  stay 0, i.e. no check fires, and the results match the oracle as in the
  release build.
"""
import ctypes
import os
import subprocess
import sys

import pytest
import torch

from tests.test_debug_build import debug_lib_path, load_with_signatures

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_index_check_selftest(cuda_ok):
    from sparse_spatiotemporal_attention_video_b200._lib import STA_DEV_DEBUG, STA_OK
    lib = load_with_signatures(debug_lib_path())
    stream = torch.cuda.current_stream().cuda_stream
    buf = torch.zeros(64, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for index in (64, -1, 1 << 30):
        assert lib.sta_selftest_index_check(buf.data_ptr(), 64, index, st.data_ptr(),
                                            stream) == STA_OK
        torch.cuda.synchronize()
        assert int(st.item()) == STA_DEV_DEBUG
        assert int(buf.abs().sum()) == 0
        st.zero_()
    assert lib.sta_selftest_index_check(buf.data_ptr(), 64, 63, st.data_ptr(), stream) == STA_OK
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert buf[63].item() == 1 and int(buf[:63].abs().sum()) == 0


def test_parity_suite_under_the_debug_build(cuda_ok):
    debug_lib_path()
    env = dict(os.environ, STA_LIB="debug")
    check = ("from sparse_spatiotemporal_attention_video_b200 import sta_debug_build; "
             "assert sta_debug_build()")
    subprocess.run([sys.executable, "-c", check], cwd=ROOT, env=env, check=True)
    files = ["tests/test_gpu_radial.py", "tests/test_gpu_attention.py", "tests/test_gpu_routed.py",
             "tests/test_gpu_entropy.py", "tests/test_gpu_dynrad.py", "tests/test_gpu_tra_token.py",
             "tests/test_gpu_tile_major.py", "tests/test_gpu_ibcs.py"]
    # the HunyuanVideo-size IBCS cases run in the release suite only (time)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu",
                        "-p", "no:cacheprovider", "-k", "not hunyuan", *files],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0, tail
