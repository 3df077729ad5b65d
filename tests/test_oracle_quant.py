"""Pins of the oracle quantizer against what the pages and mathematics fix.

* shrinkage bias closed form (l_i - r_i)/2 for x uniform on a level's RTNE bin,
  zero on the uniform grid: "Ripensare il Bias di Shrinkage nel Pretraining di
  LLM in FP4", Metodologia 1 and 2 (fixture tests/golden/shrinkage_bias.txt);
* E[SR(x)] = x: "TetraJet-v2", section 2.A (unbiased gradient estimation);
* identity on representable values, brute force over all codes on tiny blocks;
* MXFP4 scale 2^(floor(log2 amax) - 2) ("Pre-addestramento ... con MXFP4");
* NVFP4 / double block invariants ("TetraJet-v2", 2.A Structure).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden

G = np.array(oracle.E2M1_GRID)


def deq(q):
    return oracle.dequantize(q)


def mx_anchor_rows(values, anchor=4.0):
    """Rows of 32 elements: an anchor that fixes the MX scale to 1, then 31 values."""
    v = np.asarray(values, np.float32)
    n = -(-len(v) // 31)
    x = np.zeros((n, 32), np.float32)
    x[:, 0] = anchor
    flat = np.zeros(n * 31, np.float32)
    flat[:len(v)] = v
    flat[len(v):] = v[0] if len(v) else 0
    x[:, 1:] = flat.reshape(n, 31)
    return x


def ufp4_rows(values):
    """Rows of 16: anchor 7 fixes the block scale to 1 when s_t = 1 (amax 3136)."""
    v = np.asarray(values, np.float32)
    n = -(-len(v) // 15)
    x = np.zeros((n, 16), np.float32)
    x[:, 0] = 7.0
    flat = np.full(n * 15, v[0], np.float32)
    flat[:len(v)] = v
    x[:, 1:] = flat.reshape(n, 15)
    return x


@pytest.mark.parametrize("row", read_golden("shrinkage_bias.txt"))
def test_shrinkage_bias_closed_form(row):
    grid, level, l, r, want = row[0], float(row[1]), float(row[2]), float(row[3]), float(row[4])
    rng = np.random.default_rng(int(level * 100))
    n = 400_000
    xs = rng.uniform(level - l, level + r, n).astype(np.float32)
    if grid == "e2m1":
        x = mx_anchor_rows(xs)
        q = oracle.quantize(x, oracle.MXFP4, axis=1)
        assert (q["scales"] == 127).all()
        got = deq(q)[:, 1:].ravel()[:n]
    else:
        x = ufp4_rows(xs)
        q = oracle.quantize(x, oracle.UFP4, axis=1, amax=3136.0)
        assert q["tensor_scale"] == 1.0 and (q["scales"] == 0x38).all()
        got = deq(q)[:, 1:].ravel()[:n]
    err = got - xs.astype(np.float64)
    assert (got == level).mean() > 0.999       # the bin maps to its level (ties aside)
    sigma = err.std() / math.sqrt(n)
    assert abs(err.mean() - want) <= 5 * sigma + 1e-12, (err.mean(), want, sigma)


SR_POINTS = [1.0, 3.0, 0.25, 1.25, 2.5, 5.0, 2.0 + 1e-4, 4.0 - 3e-4, 0.1234567, 5.4321]


@pytest.mark.parametrize("xv", SR_POINTS)
def test_sr_unbiased_e2m1(xv):
    n = 10_000_000
    x = mx_anchor_rows(np.full(n, xv, np.float32))
    q = oracle.quantize(x, oracle.MXFP4, rounding=oracle.SR, axis=1, seed=0xC0FFEE, tensor_id=7)
    got = deq(q)[:, 1:].ravel()[:n]
    xv32 = float(np.float32(xv))
    lo = G[G <= xv32].max()
    hi = G[G > xv32].min() if xv32 < 6 else lo
    assert set(np.unique(got)) <= {lo, hi}
    if xv32 in G:
        assert (got == xv32).all()
        return
    sigma = got.std() / math.sqrt(n)
    assert abs(got.mean() - xv32) <= 5 * sigma + 2.0 ** -24 * (hi - lo)
    # it really is stochastic: the up-fraction follows the position in the bin
    f = (xv32 - lo) / (hi - lo)
    assert abs((got == hi).mean() - f) <= 5 * math.sqrt(f * (1 - f) / n) + 1e-6


@pytest.mark.parametrize("xv", [2.0, 2.5, 3.3333, 6.75, 0.01])
def test_sr_unbiased_ufp4(xv):
    n = 3_000_000
    x = ufp4_rows(np.full(n, xv, np.float32))
    q = oracle.quantize(x, oracle.UFP4, rounding=oracle.SR, axis=1, amax=3136.0, seed=5)
    got = deq(q)[:, 1:].ravel()[:n]
    xv32 = float(np.float32(xv))
    if xv32 == int(xv32):
        assert (got == xv32).all()
        return
    sigma = got.std() / math.sqrt(n)
    assert abs(got.mean() - xv32) <= 5 * sigma + 2.0 ** -24


def test_sr_reproducible_and_stream_separated():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    a = oracle.quantize(x, oracle.MXFP4, rounding=oracle.SR, seed=11, tensor_id=1)
    b = oracle.quantize(x, oracle.MXFP4, rounding=oracle.SR, seed=11, tensor_id=1)
    c = oracle.quantize(x, oracle.MXFP4, rounding=oracle.SR, seed=11, tensor_id=2)
    d = oracle.quantize(x, oracle.MXFP4, rounding=oracle.SR, seed=12, tensor_id=1)
    assert (a["codes"] == b["codes"]).all()
    assert (a["codes"] != c["codes"]).any() and (a["codes"] != d["codes"]).any()
    assert (a["scales"] == c["scales"]).all()


def test_identity_on_representable_mx():
    rng = np.random.default_rng(4)
    rows = []
    for _ in range(500):
        k = int(rng.integers(-60, 60))
        row = rng.choice(G, 32) * rng.choice([-1, 1], 32)
        row[rng.integers(32)] = rng.choice([4.0, 6.0]) * rng.choice([-1, 1])
        rows.append(row * 2.0 ** k)
    x = np.array(rows, np.float32)
    for rot_free_axis in (1,):
        q = oracle.quantize(x, oracle.MXFP4, axis=rot_free_axis)
        assert (deq(q) == x.astype(np.float64)).all()


def e4m3_values():
    return np.array([oracle.e4m3_value(c) for c in range(1, 0x7F)])


def test_identity_on_representable_nv_and_ufp4():
    rng = np.random.default_rng(5)
    E = e4m3_values()
    for fmt, grid, top in ((oracle.NVFP4, G, 6.0), (oracle.UFP4, np.arange(8.0), 7.0)):
        rows = []
        for _ in range(400):
            e = rng.choice(E)
            row = rng.choice(grid, 16) * rng.choice([-1, 1], 16)
            row[rng.integers(16)] = top * rng.choice([-1, 1])
            rows.append(row * e)
        x = np.array(rows, np.float32)
        amax = float(top * 448)          # s_t = 1 exactly
        q = oracle.quantize(x, fmt, axis=1, amax=amax)
        assert q["tensor_scale"] == 1.0
        assert (deq(q) == x.astype(np.float64)).all()


def test_identity_on_representable_double_block():
    rng = np.random.default_rng(6)
    E = e4m3_values()
    rows = []
    for _ in range(200):
        j = int(rng.integers(-20, 20))
        s_o = 2.0 ** j
        row = np.zeros(128)
        for b in range(8):
            e = rng.choice(E[E <= 448])
            blk = rng.choice(G, 16) * rng.choice([-1, 1], 16)
            blk[rng.integers(16)] = 6.0
            row[16 * b:16 * b + 16] = blk * e * s_o
        # plant the chunk max 2688 * 2^j (so s_o = 2^j exactly) alone in its block,
        # which then has E = 448 and stays representable
        p = int(rng.integers(128))
        row[16 * (p // 16):16 * (p // 16) + 16] = 0.0
        row[p] = 2688.0 * s_o * rng.choice([-1, 1])
        rows.append(row)
    x = np.array(rows, np.float32)
    q = oracle.quantize(x, oracle.NVFP4, axis=1, double_block=True)
    assert (q["outer"] == np.float32(2.0) ** np.round(np.log2(q["outer"]))).all()
    assert (deq(q) == x.astype(np.float64)).all()


def brute_codes(x_block, S, grid):
    """Nearest dequantized value q*S over all 16 codes, ties to the even magnitude."""
    out = []
    for xv in x_block.astype(np.float64):
        d = [abs(xv - (-1) ** (c >> 3) * grid[c & 7] * S) for c in range(16)]
        best = min(d)
        cands = [c for c in range(16) if d[c] == best]
        # sign follows x; among equal distances the even magnitude
        sgn = 8 if np.signbit(xv) else 0
        mags = sorted(set(c & 7 for c in cands))
        m = mags[0] if len(mags) == 1 else [v for v in mags if v % 2 == 0][0]
        out.append(sgn | m)
    return out


def unpack(codes, K):
    c = np.zeros((codes.shape[0], K), np.uint8)
    c[:, 0::2] = codes & 0xF
    c[:, 1::2] = codes >> 4
    return c


def test_brute_force_mx_blocks():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((40, 64)) * 10.0 ** rng.uniform(-3, 3, (40, 1))).astype(np.float32)
    q = oracle.quantize(x, oracle.MXFP4, axis=1)
    codes = unpack(q["codes"], 64)
    for r in range(40):
        for b in range(2):
            blk = x[r, 32 * b:32 * b + 32]
            m = np.abs(blk).max()
            e = math.frexp(float(m))[1] - 1 - 2
            assert q["scales"][r, b] == e + 127
            assert 4.0 <= m / 2.0 ** e < 8.0
            assert list(codes[r, 32 * b:32 * b + 32]) == brute_codes(blk, 2.0 ** e, G)


def test_brute_force_nv_blocks_and_tensor_scale():
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((40, 64)) * 3).astype(np.float32)
    x[3, 5] = 250.0
    q = oracle.quantize(x, oracle.NVFP4, axis=1)
    assert q["amax"] == 250.0
    s_t = q["tensor_scale"]
    assert abs(s_t - 250.0 / 2688.0) <= 2.0 ** -24 * s_t
    codes = unpack(q["codes"], 64)
    for r in range(40):
        for b in range(4):
            blk = x[r, 16 * b:16 * b + 16]
            E = q["scales"][r, b]
            sb = np.float32(np.float32(np.abs(blk).max() / np.float32(6)) / np.float32(s_t))
            assert E == torch.tensor([float(sb)]).to(torch.float8_e4m3fn).view(torch.uint8).item()
            S = float(np.float32(oracle.e4m3_value(E) * np.float32(s_t)))
            assert list(codes[r, 16 * b:16 * b + 16]) == brute_codes(blk, S, G)
    # the block holding the tensor amax is scaled to the top: E = 448, element -> 6
    assert q["scales"][3, 0] == 0x7E and codes[3, 5] == 7


def test_axis0_is_axis1_of_transpose_rtne():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((96, 40)).astype(np.float32)
    for fmt, rot in ((oracle.MXFP4, oracle.ROT_H32), (oracle.NVFP4, oracle.ROT_H16),
                     (oracle.UFP4, oracle.ROT_RH16), (oracle.MXFP4, oracle.ROT_NONE)):
        a = oracle.quantize(x, fmt, rotation=rot, axis=0, seed=3)
        b = oracle.quantize(np.ascontiguousarray(x.T), fmt, rotation=rot, axis=1, seed=3)
        assert (a["codes"] == b["codes"]).all() and (a["scales"] == b["scales"]).all()
        assert a["amax"] == b["amax"]


def test_bf16_input_equals_float32_input():
    rng = np.random.default_rng(10)
    xf = torch.from_numpy(rng.standard_normal((32, 64)).astype(np.float32)).to(torch.bfloat16)
    bits = xf.view(torch.int16).numpy().view(np.uint16)
    f32 = xf.to(torch.float32).numpy()
    for fmt in (oracle.MXFP4, oracle.NVFP4):
        a = oracle.quantize(bits, fmt, rotation=oracle.ROT_H16, rounding=oracle.SR, seed=1)
        b = oracle.quantize(f32, fmt, rotation=oracle.ROT_H16, rounding=oracle.SR, seed=1)
        assert (a["codes"] == b["codes"]).all() and (a["scales"] == b["scales"]).all()


def test_ld_padding_is_ignored():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((64, 48)).astype(np.float32)
    padded = np.full((64, 56), 1e30, np.float32)
    padded[:, :48] = x
    a = oracle.quantize(x, oracle.NVFP4, axis=0, rounding=oracle.SR, seed=4)
    b = oracle.quantize(padded, oracle.NVFP4, axis=0, rounding=oracle.SR, seed=4, C=48)
    assert (a["codes"] == b["codes"]).all() and (a["scales"] == b["scales"]).all()


def test_zero_blocks_and_negative_zero():
    x = np.zeros((2, 32), np.float32)
    x[1, :] = -0.0
    q = oracle.quantize(x, oracle.MXFP4)
    assert (q["scales"] == 0).all()
    assert (q["codes"][0] == 0).all() and (q["codes"][1] == 0x88).all()
    q = oracle.quantize(x[:, :16].copy(), oracle.NVFP4)
    assert q["tensor_scale"] == 1.0 and (q["scales"] == 0).all()
    assert (q["codes"][1] == 0x88).all()
    # small negatives that round to zero keep their sign bit
    y = np.full((1, 32), -0.01, np.float32)
    y[0, 0] = 4.0
    c = unpack(oracle.quantize(y, oracle.MXFP4)["codes"], 32)
    assert (c[0, 1:] == 8).all()


def test_rotation_changes_amax_and_matches_manual_blocks():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((8, 64)).astype(np.float32)
    x[2, 7] = 100.0
    amax = oracle.tensor_amax(x, 1, oracle.ROT_H16)
    manual = max(np.abs(oracle.rotate_block(x[r, 16 * b:16 * b + 16])).max()
                 for r in range(8) for b in range(4))
    assert amax == manual and amax < 100.0


def test_underflowing_scales_fall_back_to_one():
    """A tensor or outer scale amax/2688 that underflows to 0 is read as 1,
    like the all-zero block: the codes are then signed zeros."""
    tiny = np.float32(2.0 ** -149)
    assert oracle.tensor_scale(float(tiny), oracle.NVFP4) == 1.0
    assert oracle.tensor_scale(0.0, oracle.UFP4) == 1.0
    x = np.full((2, 128), tiny, np.float32)
    x[1] *= -1
    q = oracle.quantize(x, oracle.NVFP4, double_block=True)
    assert (q["outer"] == 1.0).all() and (q["scales"] == 0).all()
    assert (q["codes"][0] == 0).all() and (q["codes"][1] == 0x88).all()
    q = oracle.quantize(x, oracle.NVFP4)
    assert q["tensor_scale"] == 1.0 and (q["scales"] == 0).all()
