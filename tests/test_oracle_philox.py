"""Pin the oracle's Philox4x32-10 against an independent implementation:
cuRAND's host-side PHILOX4_32_10 generator (runs on the CPU, no GPU needed).

With the default ordering, output group j (four 32-bit words) of the host
generator seeded with s and offset o*4 is Philox4x32-10 with key
(lo32(s), hi32(s)) and counter (lo32(q // 65536), hi32(q // 65536), q % 65536, 0),
q = j + o.  That exercises counter words 0, 1, 2 and both key words.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle

CURAND = "/usr/local/cuda/lib64/libcurand.so"
PHILOX = 161  # CURAND_RNG_PSEUDO_PHILOX4_32_10


def curand_host(seed, offset_groups, ngroups):
    cr = ctypes.CDLL(CURAND)
    g = ctypes.c_void_p()
    assert cr.curandCreateGeneratorHost(ctypes.byref(g), PHILOX) == 0
    try:
        assert cr.curandSetPseudoRandomGeneratorSeed(g, ctypes.c_ulonglong(seed)) == 0
        assert cr.curandSetGeneratorOffset(g, ctypes.c_ulonglong(offset_groups * 4)) == 0
        out = np.zeros(ngroups * 4, np.uint32)
        assert cr.curandGenerate(g, out.ctypes.data_as(ctypes.c_void_p),
                                 ctypes.c_size_t(out.size)) == 0
    finally:
        cr.curandDestroyGenerator(g)
    return out.reshape(-1, 4)


pytestmark = pytest.mark.skipif(not os.path.exists(CURAND), reason="libcurand not found")


@pytest.mark.parametrize("seed", [0, 1, 0x123456789ABCDEF, 0xFEDCBA9876543210, 2**64 - 1])
def test_philox_matches_curand_host(seed):
    key = [seed & 0xFFFFFFFF, seed >> 32]
    rng = np.random.default_rng(seed & 0xFFFF)
    for off in [0, 65536 * 3 + 17, (1 << 48) + 5, (1 << 52) + 65536 * 7 + 3,
                int(rng.integers(0, 1 << 60))]:
        grp = curand_host(seed, off, 64)
        for j in range(64):
            q = off + j
            hi = q // 65536
            ctr = [hi & 0xFFFFFFFF, hi >> 32, q % 65536, 0]
            assert (oracle.philox4x32_10(ctr, key) == grp[j]).all(), (seed, off, j)


def test_rht_signs_are_bits_of_one_philox_word():
    for seed in (0, 7, 2**40 + 3):
        w = oracle.philox4x32_10([0, 0, 0, 1], [seed & 0xFFFFFFFF, seed >> 32])[0]
        d = oracle.rht_signs(seed, 32)
        assert ((d == -1) == np.array([(int(w) >> j) & 1 for j in range(32)], bool)).all()
        assert (oracle.rht_signs(seed, 16) == d[:16]).all()
