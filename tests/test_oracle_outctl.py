"""Pins of the oracle's OutControl split ("TetraJet-v2" 2.C: the top p% of
activation channels, chosen in a calibration window and then fixed, kept in
FP8 for the forward and backward passes, the rest in FP4).

  * channel choice: planted outlier channels are the ones chosen; equal maxima
    go to the lower index;
  * FP8 (E4M3 under one tensor scale amax / 448): identity on representable
    values, signs (-0 kept), saturation, and torch's float8_e4m3fn rounding;
  * the split GEMM: exact rational arithmetic over both parts on tiny
    operands; an empty channel set is the plain FP4 GEMM;
  * the page's claim: on activations with outlier channels the split product
    is closer to the exact product than the plain NVFP4 one.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

NV = oracle.NVFP4


def test_channels_are_the_planted_outliers():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((512, 1024)).astype(np.float32)
    planted = np.sort(rng.choice(1024, 8, replace=False))
    x[:, planted] *= 64.0
    assert (oracle.outctl_channels(x, 8 / 1024) == planted).all()
    # ceil(p * cols) channels, in ascending order
    ch = oracle.outctl_channels(x, 0.1)
    assert len(ch) == 103 and (np.diff(ch) > 0).all() and set(planted) <= set(ch)


def test_channel_ties_go_to_the_lower_index():
    x = np.ones((4, 16), np.float32)
    x[:, 9] = 2.0
    assert list(oracle.outctl_channels(x, 3 / 16)) == [0, 1, 9]


def test_fp8_identity_on_representable_values():
    codes = np.arange(0, 0x7F, dtype=np.uint8)
    vals = np.array([oracle.e4m3_value(int(c)) for c in codes], np.float32)
    s8 = 0.25                                        # a power of two: x / s8 exact
    x = np.concatenate([vals, -vals]).astype(np.float32)[None, :] * np.float32(s8)
    q = oracle.fp8_quantize(x, x.shape[1], scale=s8)
    want = np.concatenate([codes, codes | 0x80])
    want[len(codes)] = 0x80                          # -0 keeps its sign
    assert (q["codes"][0] == want).all()
    assert (oracle.fp8_dequantize(q)[0] == x[0].astype(np.float64)).all()


def test_fp8_scale_saturation_and_torch_rounding():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((64, 96)) * 3).astype(np.float32)
    q = oracle.fp8_quantize(x, 128)
    assert q["scale"] == np.float32(np.float32(np.abs(x).max()) / np.float32(448.0))
    assert (q["codes"][:, 96:] == 0).all()
    v = (x / np.float32(q["scale"])).astype(np.float32)
    ok = np.abs(v) <= 448.0
    t = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (q["codes"][:, :96][ok] == t[ok]).all()
    assert ((q["codes"][:, :96][~ok] & 0x7F) == 0x7E).all()       # saturated to 448
    big = oracle.fp8_quantize(np.array([[1e30, -1e30]], np.float32), 2, scale=1.0)
    assert list(big["codes"][0]) == [0x7E, 0xFE]


def e2m1_exact(code):
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
    return -mag if s else mag


def e4m3_exact(code):
    v = Fraction(torch.tensor([code & 0x7F], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item())
    return -v if code & 0x80 else v


@pytest.mark.parametrize("shape", [(1, 1, 32, 16), (2, 3, 64, 32)])
def test_split_gemm_brute_force(shape):
    M, N, K, K8 = shape
    rng = np.random.default_rng(sum(shape))
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    ca, cb = rng.integers(0, 16, (M, K)).astype(np.uint8), rng.integers(0, 16, (N, K)).astype(np.uint8)
    sa, sb = rng.integers(1, 0x7F, (M, K // 16)).astype(np.uint8), rng.integers(1, 0x7F, (N, K // 16)).astype(np.uint8)
    ta, tb = np.float32(0.7), np.float32(1.3)
    a8 = rng.integers(0, 255, (M, K8)).astype(np.uint8)
    b8 = rng.integers(0, 255, (N, K8)).astype(np.uint8)
    a8[(a8 & 0x7F) == 0x7F] = 0x10                  # no NaN codes
    b8[(b8 & 0x7F) == 0x7F] = 0x11
    s8a, s8b = np.float32(0.125), np.float32(3.0)
    qa = dict(fp4=dict(codes=pack(ca), scales=sa, K=K, format=NV, double_block=False, tensor_scale=float(ta),
                       outer=None), fp8=dict(codes=a8, scale=float(s8a), K=K8))
    qb = dict(fp4=dict(codes=pack(cb), scales=sb, K=K, format=NV, double_block=False, tensor_scale=float(tb),
                       outer=None), fp8=dict(codes=b8, scale=float(s8b), K=K8))
    C64, bound = oracle.gemm_outctl(qa, qb)
    for i in range(M):
        for j in range(N):
            terms = [e2m1_exact(int(ca[i, k])) * e4m3_exact(int(sa[i, k // 16])) * Fraction(float(ta)) *
                     e2m1_exact(int(cb[j, k])) * e4m3_exact(int(sb[j, k // 16])) * Fraction(float(tb)) for k in range(K)]
            terms += [e4m3_exact(int(a8[i, k])) * Fraction(float(s8a)) * e4m3_exact(int(b8[j, k])) * Fraction(float(s8b))
                      for k in range(K8)]
            exact, absb = sum(terms), sum(abs(t) for t in terms)
            assert abs(Fraction(C64[i, j]) - exact) <= Fraction(2.0 ** -50) * absb
            assert abs(Fraction(bound[i, j]) - absb) <= Fraction(2.0 ** -50) * absb


def test_empty_channel_set_is_the_fp4_gemm():
    rng = np.random.default_rng(2)
    x, w = rng.standard_normal((32, 256)).astype(np.float32), rng.standard_normal((16, 256)).astype(np.float32)
    none = np.zeros(0, np.int32)
    a, b = oracle.outctl_quantize(x, none, 128), oracle.outctl_quantize(w, none, 128)
    C, bound = oracle.gemm_outctl(a, b)
    C4, b4 = oracle.gemm(oracle.quantize(x, NV), oracle.quantize(w, NV))
    assert (C == C4).all() and (bound == b4).all()


def test_outliers_in_fp8_reduce_the_error():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((256, 1024)).astype(np.float32)
    x[:, rng.choice(1024, 8, replace=False)] *= 64.0
    w = (rng.standard_normal((128, 1024)) * 0.02).astype(np.float32)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    ch = oracle.outctl_channels(x, 0.1)
    split = oracle.gemm_outctl(oracle.outctl_quantize(x, ch, 128), oracle.outctl_quantize(w, ch, 128))[0]
    plain = oracle.gemm(oracle.quantize(x, NV), oracle.quantize(w, NV))[0]
    e_split = np.linalg.norm(split - exact) / np.linalg.norm(exact)
    e_plain = np.linalg.norm(plain - exact) / np.linalg.norm(exact)
    assert e_split < 0.7 * e_plain, (e_split, e_plain)
