"""Pins of the oracle's re-quantization ("TetraJet-v2" 2.A: the backward pass
works on X^, the dequantized forward operand, re-quantized along the
transposed axis).

- The binary32 X^ is the exact product q * s_block * s_ref rounded once to
  nearest-even (a zero keeps the code's sign).  This is checked against exact rational arithmetic built from
  the code and scale definitions, not against the oracle's own dequantizer.
- On values that MXFP4 represents exactly in both directions, re-quantizing
  along the other axis is the identity.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle

E2M1 = [Fraction(v) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]


def e4m3_exact(code):
    """E4M3 (bias 7, subnormals 2^-9 apart, no inf/nan used) as a Fraction."""
    e, m = (code >> 3) & 0xF, code & 7
    if e == 0:
        return Fraction(m, 8) * Fraction(1, 2 ** 6)
    return (1 + Fraction(m, 8)) * (Fraction(2) ** (e - 7))


def nearest_binary32(x: Fraction) -> np.float32:
    """Round a rational to the nearest binary32, ties to even, by bracketing."""
    f = np.float32(float(x))           # within one ulp of x
    lo, hi = f, f
    while Fraction(float(lo)) > x:
        lo = np.nextafter(lo, np.float32(-np.inf))
    while Fraction(float(hi)) < x:
        hi = np.nextafter(hi, np.float32(np.inf))
    if lo == hi:
        return lo
    dl, dh = x - Fraction(float(lo)), Fraction(float(hi)) - x
    if dl != dh:
        return lo if dl < dh else hi
    return lo if (int(np.float32(lo).view(np.uint32)) & 1) == 0 else hi


def code_value(c, ufp4):
    mag = Fraction(c & 7) if ufp4 else E2M1[c & 7]
    return -mag if c & 8 else mag


@pytest.mark.parametrize("fmt,db", [(oracle.MXFP4, False), (oracle.NVFP4, False), (oracle.NVFP4, True),
                                    (oracle.UFP4, False)])
def test_binary32_xhat_is_the_exact_product_rounded_once(fmt, db):
    rng = np.random.default_rng(7)
    n, K = 6, 256
    x = (rng.standard_normal((n, K)) * rng.choice([1e-3, 1.0, 37.0], (n, 1))).astype(np.float32)
    q = oracle.quantize(x, fmt, double_block=db)
    got = oracle.dequantize32(q)
    blk = 32 if fmt == oracle.MXFP4 else 16
    ts = Fraction(float(np.float32(q["tensor_scale"]))) if q["tensor_scale"] is not None else None
    for l in range(n):
        for k in range(0, K, 7):
            byte = int(q["codes"][l, k // 2])
            c = (byte >> 4) if k & 1 else (byte & 0xF)
            sb = int(q["scales"][l, k // blk])
            if fmt == oracle.MXFP4:
                s = Fraction(2) ** (sb - 127)
            else:
                ref = Fraction(float(q["outer"][l, k // 128])) if db else ts
                s = e4m3_exact(sb) * ref
            exact = code_value(c, fmt == oracle.UFP4) * s
            want = nearest_binary32(exact) if exact != 0 else np.float32(-0.0 if c & 8 else 0.0)
            assert np.float32(got[l, k]).view(np.uint32) == np.float32(want).view(np.uint32), (l, k, c, sb)


def test_requantize_is_identity_on_values_mxfp4_represents_both_ways():
    # X = 2^E[tile] * Q with Q on the E2M1 grid, and +-6 on the diagonal of
    # every 32 x 32 tile, so every 32-block along either axis has max 6 * 2^E:
    # the MX exponent is E both ways and every value is a grid point times 2^E
    rng = np.random.default_rng(3)
    R, C = 64, 96
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    Q = grid[rng.integers(0, 8, (R, C))] * rng.choice([-1.0, 1.0], (R, C))
    for r in range(R):
        Q[r, (r % 32) + 32 * np.arange(C // 32)] = 6.0 * rng.choice([-1.0, 1.0], C // 32)
    E = rng.integers(-20, 20, (R // 32, C // 32))
    X = (Q * np.exp2(np.repeat(np.repeat(E, 32, 0), 32, 1))).astype(np.float32)
    fwd = oracle.quantize(X, oracle.MXFP4, axis=1)
    assert np.array_equal(oracle.dequantize(fwd), X.astype(np.float64))
    back = oracle.requantize(fwd, oracle.MXFP4)
    assert back["codes"].shape == (C, R // 2)
    assert np.array_equal(oracle.dequantize(back), X.T.astype(np.float64))
