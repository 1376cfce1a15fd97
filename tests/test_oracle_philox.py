"""Pin for oracle.philox against cuRAND's host-side Philox4_32_10 generator,
called through cuRAND's public host API (runs on the CPU, no GPU needed).

cuRAND's host generator lays a stream position p out as counter word 0 =
(p/4) // 65536, counter word 2 = (p/4) % 65536 (its subsequence), key = the
64-bit seed split in two words, output word p % 4.  That layout was observed
from the stream itself (positions 4, 16, 400 and 262144 carry counters
(0,0,1,0), (0,0,4,0), (0,0,100,0) and (1,0,0,0)); the test re-derives every
compared value from it.
"""
import ctypes
import glob
import os

import numpy as np
import pytest

from oracle import philox

_CANDIDATES = ["/usr/local/cuda/lib64/libcurand.so.10",
               "/usr/local/cuda/targets/x86_64-linux/lib/libcurand.so.10"]
_CANDIDATES += glob.glob("/usr/local/cuda*/targets/x86_64-linux/lib/libcurand.so.10")
try:
    import nvidia.curand as _nc  # pip wheel bundled with torch
    _CANDIDATES += glob.glob(os.path.join(list(_nc.__path__)[0], "lib", "libcurand.so*"))
except Exception:
    pass


def _curand():
    for p in _CANDIDATES:
        if os.path.exists(p):
            try:
                return ctypes.CDLL(p)
            except OSError:
                continue
    pytest.skip("libcurand not found")


def _curand_stream(lib, seed, offset, n):
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0  # PHILOX4_32_10
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(offset)) == 0
        out = np.zeros(n, dtype=np.uint32)
        assert lib.curandGenerate(gen, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(n)) == 0
        return out
    finally:
        lib.curandDestroyGenerator(gen)


@pytest.mark.parametrize("seed", [0, 1, 0x0123456789ABCDEF, 0x5EED5A3C1E5B00B5, (1 << 64) - 1])
def test_philox_matches_curand_host(seed):
    lib = _curand()
    n = 1 << 19                               # covers counter word 0 in {0, 1}
    stream = _curand_stream(lib, seed, 0, n)
    p = np.arange(n, dtype=np.uint64)
    grp = p // np.uint64(4)
    c0 = grp // np.uint64(65536)
    c2 = grp % np.uint64(65536)
    outs = philox.philox4x32_10(c0, 0, c2, 0, seed & 0xFFFFFFFF, seed >> 32)
    got = np.stack(outs)[(p % np.uint64(4)).astype(np.int64), np.arange(n)]
    assert np.array_equal(got, stream)


def test_sip_words_match_curand_rows():
    lib = _curand()
    seed = 0x5EED5A3C1E5B00B5
    n_words = 64
    for row in [0, 1, 927, 22295]:
        # word j of row r sits at counter (j//4, 0, r, 0): stream position
        # 4 * ((j//4) * 65536 + r) + j % 4
        ref = []
        for j in range(n_words):
            pos = 4 * ((j // 4) * 65536 + row) + j % 4
            ref.append(_curand_stream(lib, seed, pos, 1)[0])
        assert np.array_equal(philox.sip_words(seed, row, n_words), np.array(ref, np.uint32))


def test_uniforms_are_24_bit_grid_in_unit_interval():
    u = philox.sip_uniforms(7, 3, 5000)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert np.array_equal(u * 2 ** 24, np.floor(u * 2 ** 24))
    assert abs(u.mean() - 0.5) < 0.02
