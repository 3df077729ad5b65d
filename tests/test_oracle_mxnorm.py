"""Pins of the oracle's MXNorm ("MXNorm: Reusing MXFP block scales for
efficient tensor normalisation", 2. Metodologia; 3. Contributi Chiave):
rho_t = c(p, B) * ((1/K) sum_k m_tk^p)^(-1/p) from the block maxima m_tk, and
the cast of y = x * rho_t.

What fixes each part, other than the oracle itself:
  * c(p, B): closed forms at B = 1 (E|z| = sqrt(2/pi), E z^2 = 1) and, for
    B = 16, 32, the page's own method, a Monte Carlo estimate;
  * the binary64 pairwise sum: a hand-derived case whose pairwise result
    differs from the sequential one, and exact integer sums;
  * rho: rows whose blocks share one maximum m give exactly RN(c / m);
    scaling x by 2^k scales rho by 2^-k and leaves the codes unchanged;
    an all-zero row gives rho = 1;
  * the page's claims: with p = 2, |y| <= c sqrt(K) (the bound that keeps
    the output limited like RMSNorm's); rho tends to 1 / RMS on long
    Gaussian rows (Theorem 1).
"""
import math

import numpy as np
import pytest

import oracle

MX, NV = oracle.MXFP4, oracle.NVFP4


def test_constant_closed_forms_at_block_1():
    assert math.isclose(oracle.mxnorm_constant(1, 1), math.sqrt(2 / math.pi), rel_tol=1e-12)
    assert math.isclose(oracle.mxnorm_constant(2, 1), 1.0, rel_tol=1e-12)


@pytest.mark.parametrize("p", [1, 2])
@pytest.mark.parametrize("B", [16, 32])
def test_constant_matches_monte_carlo(p, B):
    rng = np.random.default_rng(100 * p + B)
    n = 400_000
    m = np.abs(rng.standard_normal((n, B))).max(axis=1) ** p
    est, se = m.mean(), m.std() / math.sqrt(n)
    quad = oracle.mxnorm_constant(p, B) ** p
    assert abs(quad - est) < 5 * se, (quad, est, se)


def test_pairwise_sum_order():
    # sequentially 2^53 absorbs every 1 (ties to even); pairwise, (1 + 1) and
    # (1 + 0) first: (2^53 + 1) + 2 = 2^53 + 2, then + 1 ties to 2^53 + 4
    a = [2.0 ** 53, 1.0, 1.0, 1.0, 1.0, 0.0, 0.0, 0.0]
    assert oracle.pairwise_sum(a) == 2.0 ** 53 + 4
    seq = 0.0
    for v in a:                                     # the sequential order differs
        seq = seq + v
    assert seq == 2.0 ** 53
    b = [2.0 ** 53, 1.0, 1.0, 1.0, 1.0]             # split 4 + 1: the same tree
    assert oracle.pairwise_sum(b) == 2.0 ** 53 + 4
    ints = np.arange(1, 1001, dtype=np.float64)
    assert oracle.pairwise_sum(ints) == 500500.0


def uniform_max_rows(m, B, K, rng):
    """Rows of K blocks whose maximum |x| is exactly m in every block."""
    x = (rng.uniform(-1, 1, (3, K * B)) * m * 0.9).astype(np.float32)
    x[:, ::B] = m
    x[1, 5::B] = -m
    return x


@pytest.mark.parametrize("p", [1, 2])
@pytest.mark.parametrize("B,m", [(32, 4.0), (16, 0.125), (32, 3.0)])
def test_rho_of_equal_block_maxima(p, B, m):
    c = 2.3
    x = uniform_max_rows(np.float32(m), B, 24, np.random.default_rng(B))
    rho, rmax = oracle.mxnorm_rho(x, B, p, c)
    assert (rho == np.float32(c / m)).all(), (rho, np.float32(c / m))
    assert (rmax == np.float32(m)).all()


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("p", [1, 2])
def test_scale_equivariance(fmt, p):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((16, 512)).astype(np.float32)
    c = oracle.mxnorm_constant(p, 32 if fmt == MX else 16)
    a = oracle.mxnorm(x, fmt, p, c)
    b = oracle.mxnorm((x * np.float32(2.0 ** 9)).astype(np.float32), fmt, p, c)
    assert (b["rho"] * np.float32(2.0 ** 9) == a["rho"]).all()
    assert (a["codes"] == b["codes"]).all() and (a["scales"] == b["scales"]).all()
    assert (a["y"] == b["y"]).all()


def test_zero_row():
    x = np.zeros((2, 64), np.float32)
    x[1, 3] = 1.0
    q = oracle.mxnorm(x, MX, 2, 2.0)
    assert q["rho"][0] == 1.0 and (q["codes"][0] == 0).all()


@pytest.mark.parametrize("fmt", [MX, NV])
def test_p2_output_bound(fmt):
    # m_max^2 <= sum_k m_k^2, so m_max * rho <= c * sqrt(K): one huge outlier
    # cannot push the normalised values past that, unlike p = 1
    B = 32 if fmt == MX else 16
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 64 * B)).astype(np.float32) * 1e-3
    x[0, 17] = 1e4
    x[1, :] = 0.0
    x[1, 5] = 1.0
    x[2, ::B] = 7.0
    c = oracle.mxnorm_constant(2, B)
    q = oracle.mxnorm(x, fmt, 2, c)
    assert np.abs(q["y"]).max() <= c * math.sqrt(64) * (1 + 1e-6)


@pytest.mark.parametrize("p", [1, 2])
def test_rho_tends_to_inverse_rms(p):
    rng = np.random.default_rng(11)
    sigma = 3.0
    x = (rng.standard_normal((4, 32 * 4096)) * sigma).astype(np.float32)
    rho, _ = oracle.mxnorm_rho(x, 32, p, oracle.mxnorm_constant(p, 32))
    rms = np.sqrt((x.astype(np.float64) ** 2).mean(axis=1))
    assert np.abs(rho * rms - 1.0).max() < 0.01, rho * rms
