"""Pin the oracle's Philox4x32-10 where cuRAND's host generator cannot: counter
word 3, and the counter (0, 0, 0, 1) that the random-sign Hadamard draws its
signs from.

cuRAND's device API (curand_init with a Philox state; a library routine run on
the GPU) places the subsequence in counter words 2-3 and offset / 4 in words
0-1, so subsequences of 2^32 and above set word 3.  Each draw is compared with
oracle.philox4x32_10 on the same key and counter, and the oracle's sign vector
of the random-sign H16 / H32 with bit j of word 0 of cuRAND's draw at
subsequence 2^32 (counter (0, 0, 0, 1)).  The helper (tests/curand/
philox_draw.cu) is built with nvcc when the test runs.
"""
import ctypes
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.fixture(scope="module")
def draw(cuda_device):
    d = tempfile.mkdtemp(prefix="philox_draw_")
    so = os.path.join(d, "philox_draw.so")
    subprocess.check_call([NVCC, "-shared", "-Xcompiler", "-fPIC", "-O2",
                           "-gencode", "arch=compute_100a,code=sm_100a",
                           os.path.join(HERE, "curand", "philox_draw.cu"), "-o", so])
    lib = ctypes.CDLL(so)
    P = ctypes.c_void_p
    lib.philox_draw.argtypes = [P, P, P, P, ctypes.c_int]

    def run(seeds, subs, groups):
        s = np.ascontiguousarray(seeds, np.uint64)
        u = np.ascontiguousarray(subs, np.uint64)
        g = np.ascontiguousarray(groups, np.uint64)
        out = np.zeros((len(s), 4), np.uint32)
        rc = lib.philox_draw(s.ctypes.data, u.ctypes.data, g.ctypes.data, out.ctypes.data, len(s))
        assert rc == 0, "cuda error %d" % rc
        return out

    yield run
    shutil.rmtree(d, ignore_errors=True)


def cases():
    rng = np.random.default_rng(3)
    seeds = [0, 1, 7, 2**40 + 3, 0xFEDCBA9876543210, 2**64 - 1] + [int(v) for v in rng.integers(0, 2**63, 4)]
    subs = [2**32, 2**32 + 5, 3 << 32, (2**64 - 1), 0x123456789ABCDEF0, 1, 0] + \
           [int(v) for v in rng.integers(2**32, 2**63, 3)]
    groups = [0, 1, 2**32 - 1, 2**40 + 17, int(rng.integers(0, 2**60))]
    out = [(s, u, g) for s in seeds for u in subs for g in groups]
    return [c[0] for c in out], [c[1] for c in out], [c[2] for c in out]


def test_oracle_philox_matches_curand_device_api_with_counter_word3(draw):
    seeds, subs, groups = cases()
    got = draw(seeds, subs, groups)
    n_word3 = 0
    for i, (s, u, g) in enumerate(zip(seeds, subs, groups)):
        ctr = [g & 0xFFFFFFFF, g >> 32, u & 0xFFFFFFFF, u >> 32]
        key = [s & 0xFFFFFFFF, s >> 32]
        n_word3 += ctr[3] != 0
        assert (oracle.philox4x32_10(ctr, key) == got[i]).all(), (s, u, g, got[i])
    assert n_word3 > 300


@pytest.mark.parametrize("n", [16, 32])
def test_random_signs_are_word0_of_curand_counter_0001(draw, n):
    seeds = [0, 3, 7, 11, 2**40 + 3, 0x5EED, 2**64 - 1]
    got = draw(seeds, [2**32] * len(seeds), [0] * len(seeds))
    for i, s in enumerate(seeds):
        want = np.array([-1.0 if (int(got[i][0]) >> j) & 1 else 1.0 for j in range(n)], np.float32)
        assert (oracle.rht_signs(s, n) == want).all(), s
