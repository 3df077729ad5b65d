"""Pin the oracle's rotation: the Sylvester Hadamard matrix from scipy (a
library construction), H H^T = n I, the binary32 butterfly against the
float64 matrix product, and the rotation applied twice giving back x.

Rotation source: "Pre-addestramento di Modelli Linguistici di Grandi
Dimensioni con MXFP4", Metodologia (deterministic H16 / H32, randomised
Hadamard); random signs on all GEMMs: "Ripensare il Bias di Shrinkage",
Metodologia 2.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle


@pytest.mark.parametrize("n", [16, 32])
def test_sylvester_orthogonality_and_entries(n):
    H = scipy.linalg.hadamard(n)
    assert (H @ H.T == n * np.eye(n)).all()
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    popc = np.vectorize(lambda v: bin(v).count("1"))(i & j)
    assert (H == (-1) ** popc).all()


@pytest.mark.parametrize("n", [16, 32])
@pytest.mark.parametrize("random_signs", [False, True])
def test_butterfly_equals_matrix_product(n, random_signs):
    rng = np.random.default_rng(n + random_signs)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    d = oracle.rht_signs(12345, n) if random_signs else None
    for _ in range(200):
        x = (rng.standard_normal(n) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32)
        y = oracle.rotate_block(x, d)
        xd = x.astype(np.float64) * (d if d is not None else 1.0)
        ref = (H @ xd) / np.sqrt(n)
        # log2(n) binary32 add stages + one multiply, each <= 2^-24 relative
        tol = (np.log2(n) + 2) * 2.0 ** -24 * np.abs(x).astype(np.float64).sum()
        assert np.abs(y - ref).max() <= tol


@pytest.mark.parametrize("n", [16, 32])
def test_rotation_is_an_involution(n):
    rng = np.random.default_rng(3)
    x = rng.standard_normal(n).astype(np.float32)
    y = oracle.rotate_block(oracle.rotate_block(x))
    assert np.abs(y - x).max() <= 1e-5 * np.abs(x).max()
    # with random signs: D H D^-1... undo is H then signs
    d = oracle.rht_signs(99, n)
    y = oracle.rotate_block(x, d)
    back = oracle.rotate_block(y) * d
    assert np.abs(back - x).max() <= 1e-5 * np.abs(x).max()


def test_h16_scale_is_exact_quarter():
    x = np.zeros(16, np.float32)
    x[0] = 1.0
    assert (oracle.rotate_block(x) == 0.25).all()
