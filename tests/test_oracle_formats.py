"""Pins of the oracle's number formats against definitions and library routines.

E2M1: the bit-field definition (2 exponent bits with bias 1, 1 mantissa bit)
from "Ripensare il Bias di Shrinkage nel Pretraining di LLM in FP4",
Problematica; E4M3 against torch.float8_e4m3fn (a library codec); E8M0 from
its power-of-two definition.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden


def e2m1_from_bits(code):
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_e2m1_grid_golden_and_bitfields():
    rows = read_golden("e2m1_grid.txt")
    assert [float(v) for _, v in rows] == list(oracle.E2M1_GRID)
    for code in range(16):
        assert oracle.e2m1_value(code) == e2m1_from_bits(code)
        assert oracle.e2m1_value(code) == (-1) ** (code >> 3) * float(rows[code & 7][1])


def test_e2m1_spacing_is_nonuniform():
    g = oracle.E2M1_GRID
    gaps = sorted(set(b - a for a, b in zip(g, g[1:])))
    assert gaps == [0.5, 1.0, 2.0]


def test_e2m1_rtne_ties_golden():
    for mid, want in read_golden("e2m1_rtne_ties.txt"):
        u = float(mid)
        assert oracle.e2m1_rtne_index(u) == int(want), mid
        # just off the tie the nearest level wins
        below = float(np.nextafter(np.float32(u), np.float32(0)))
        above = float(np.nextafter(np.float32(u), np.float32(10)))
        g = oracle.E2M1_GRID
        lo = max(k for k in range(8) if g[k] < u)
        assert oracle.e2m1_rtne_index(below) == lo
        assert oracle.e2m1_rtne_index(above) == lo + 1


def test_e2m1_rtne_brute_force_and_saturation():
    rng = np.random.default_rng(1)
    g = np.array(oracle.E2M1_GRID)
    for u in rng.uniform(0, 8, 4000).astype(np.float32):
        uu = min(float(u), 6.0)
        d = np.abs(g - uu)
        cand = np.flatnonzero(d == d.min())
        want = cand[0] if len(cand) == 1 else [k for k in cand if k % 2 == 0][0]
        assert oracle.e2m1_rtne_index(float(u)) == want
    assert oracle.e2m1_rtne_index(1e30) == 7


def test_ufp4_rtne_ties_golden():
    for mid, want in read_golden("ufp4_rtne_ties.txt"):
        assert oracle.ufp4_rtne_index(float(mid)) == int(want)
    for k in range(8):
        assert oracle.ufp4_rtne_index(float(k)) == k
        assert oracle.ufp4_value(k) == k and oracle.ufp4_value(8 | k) == -k
    assert oracle.ufp4_rtne_index(100.0) == 7


def test_e4m3_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(v)
        else:
            assert v == ref[c], c


def test_e4m3_encode_matches_torch_rne():
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    mids = [(a + b) / 2 for a, b in zip(vals, vals[1:])]
    rng = np.random.default_rng(2)
    xs = np.concatenate([np.array(vals), np.array(mids),
                         np.nextafter(np.array(mids, np.float32), 0),
                         np.nextafter(np.array(mids, np.float32), 1e9),
                         rng.uniform(0, 448, 3000), 2.0 ** rng.uniform(-14, 8.8, 3000)]).astype(np.float32)
    xs = xs[(xs >= 0) & (xs <= 448)]
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(x)) for x in xs], dtype=np.uint8)
    bad = np.flatnonzero(got != ref)
    assert len(bad) == 0, (xs[bad][:5], got[bad][:5], ref[bad][:5])


def test_e4m3_encode_saturates():
    for x in (448.0, 449.0, 463.9, 464.0, 500.0, 1e6, 3.0e38):
        assert oracle.e4m3_encode(x) == 0x7E
    assert oracle.e4m3_encode(0.0) == 0
    assert oracle.e4m3_encode(2.0 ** -10) == 0          # tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(1.5 * 2.0 ** -10) == 1


def test_c32_is_nearest_binary32_to_inv_sqrt32():
    from fractions import Fraction
    c = np.float32(oracle.c32())
    lo, hi = np.nextafter(c, np.float32(0)), np.nextafter(c, np.float32(1))
    # compare squares to avoid irrational arithmetic: t = 1/sqrt(32) <=> t^2 = 1/32
    mid_lo = (Fraction(float(lo)) + Fraction(float(c))) / 2
    mid_hi = (Fraction(float(c)) + Fraction(float(hi))) / 2
    assert mid_lo ** 2 < Fraction(1, 32) < mid_hi ** 2
    assert c.view(np.uint32) == 0x3E3504F3
