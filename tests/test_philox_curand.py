"""The oracle's Philox4x32-10 against an independent implementation: cuRAND's host generator
(CURAND_RNG_PSEUDO_PHILOX4_32_10, called as a library routine on the CPU).  Its output stream
places block j at counter (0, 0, j, 0) under key (seed low 32 bits, seed high 32 bits), the
subsequence word of curand_init, so every block of the stream must equal the oracle's block
function at that counter."""

import ctypes as ct
import ctypes.util
import os

import numpy as np
import pytest

PHILOX4_32_10 = 161  # curandRngType_t value of the Philox generator


def curand():
    for name in ("/usr/local/cuda/lib64/libcurand.so.10", ctypes.util.find_library("curand")):
        if name and (os.path.sep not in name or os.path.exists(name)):
            try:
                return ct.CDLL(name)
            except OSError:
                continue
    pytest.skip("libcurand is not available")


@pytest.mark.parametrize("seed", [0, 0x0123456789ABCDEF, 0xF1A54EAD, 0xFFFFFFFFFFFFFFFF])
def test_oracle_philox_equals_curand_stream(orc, seed):
    cr = curand()
    g = ct.c_void_p()
    assert cr.curandCreateGeneratorHost(ct.byref(g), PHILOX4_32_10) == 0
    try:
        assert cr.curandSetPseudoRandomGeneratorSeed(g, ct.c_ulonglong(seed)) == 0
        n = 1 << 14
        out = np.zeros(n, dtype=np.uint32)
        assert cr.curandGenerate(g, out.ctypes.data_as(ct.c_void_p), ct.c_size_t(n)) == 0
    finally:
        cr.curandDestroyGenerator(g)
    L = orc.lib()
    key = (ct.c_uint32 * 2)(seed & 0xFFFFFFFF, seed >> 32)
    got = (ct.c_uint32 * 4)()
    for j in range(n // 4):
        L.orc_philox4x32_10((ct.c_uint32 * 4)(0, 0, j, 0), key, got)
        assert list(got) == out[4 * j:4 * j + 4].tolist(), j
