"""Pin the GEMM oracle (dequantize exactly, float64 product) against exact
rational arithmetic on tiny operands that enumerate every 4-bit code.

The GEMM is C[i, j] = sum_k deq(A)[i, k] * deq(B)[j, k] for A [M, K] and
B [N, K] quantized along K ("Pre-addestramento ... con MXFP4", Metodologia:
FP4 operands in the Fprop / Dgrad / Wgrad GEMMs; block scales per 32 (MX) or
16 (NV, UFP4) elements, "TetraJet-v2" 2.A for the 16-groups and 128/16 double
block; the uniform UFP4 levels of "Ripensare il Bias di Shrinkage nel
Pretraining di LLM in FP4", Metodologia 2).
Codes are packed here by hand, element 2j in the low nibble of byte j.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def e2m1_exact(code):
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
    return -mag if s else mag


def ufp4_exact(code):
    """UFP4 level k * sign, k = code & 7 ("Ripensare il Bias di Shrinkage...",
    Metodologia 2: levels k s, k in [-7, 7])."""
    k = Fraction(code & 7)
    return -k if code & 8 else k


def e4m3_exact(code):
    v = torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item()
    return Fraction(v)


def pack(codes):
    codes = np.asarray(codes, np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def all_code_rows(rows, K, rng):
    out = np.zeros((rows, K), np.uint8)
    for r in range(rows):
        out[r] = rng.permutation(np.tile(np.arange(16), K // 16))
    return out


@pytest.mark.parametrize("fmt,db", [(oracle.MXFP4, False), (oracle.NVFP4, False),
                                    (oracle.NVFP4, True), (oracle.UFP4, False)])
@pytest.mark.parametrize("shape", [(1, 1, 32), (2, 2, 64), (3, 2, 256)])
def test_gemm_oracle_brute_force(fmt, db, shape):
    M, N, K = shape
    if db and K % 128:
        pytest.skip("double block needs K % 128 == 0")
    rng = np.random.default_rng(M * 100 + N * 10 + K + fmt + 5 * db)
    blk = 32 if fmt == oracle.MXFP4 else 16
    ca, cb = all_code_rows(M, K, rng), all_code_rows(N, K, rng)
    if fmt == oracle.MXFP4:
        sa = rng.integers(100, 150, (M, K // blk)).astype(np.uint8)
        sb = rng.integers(100, 150, (N, K // blk)).astype(np.uint8)
        dec = lambda b: Fraction(2) ** (int(b) - 127)
    else:
        sa = rng.integers(1, 0x7F, (M, K // blk)).astype(np.uint8)
        sb = rng.integers(1, 0x7F, (N, K // blk)).astype(np.uint8)
        dec = e4m3_exact
    ta, tb = np.float32(rng.uniform(0.01, 3)), np.float32(rng.uniform(0.01, 3))
    oa = rng.uniform(0.01, 3, (M, max(K // 128, 1))).astype(np.float32)
    ob = rng.uniform(0.01, 3, (N, max(K // 128, 1))).astype(np.float32)

    def qt(codes, scales, ts, outer):
        return dict(codes=pack(codes), scales=scales, K=K, format=fmt, double_block=db,
                    tensor_scale=None if (fmt == oracle.MXFP4 or db) else float(ts),
                    outer=outer if db else None)

    C64, bound = oracle.gemm(qt(ca, sa, ta, oa), qt(cb, sb, tb, ob))

    def ref(codes, scales, ts, outer, i, k):
        elem = ufp4_exact if fmt == oracle.UFP4 else e2m1_exact
        v = elem(int(codes[i, k])) * dec(scales[i, k // blk])
        if fmt != oracle.MXFP4:
            v *= Fraction(float(outer[i, k // 128])) if db else Fraction(float(ts))
        return v

    for i in range(M):
        for j in range(N):
            terms = [ref(ca, sa, ta, oa, i, k) * ref(cb, sb, tb, ob, j, k) for k in range(K)]
            exact = sum(terms)
            absb = sum(abs(t) for t in terms)
            assert abs(Fraction(C64[i, j]) - exact) <= Fraction(2.0 ** -50) * absb
            assert abs(Fraction(bound[i, j]) - absb) <= Fraction(2.0 ** -50) * absb


def test_gemm_oracle_on_quantized_random_operands():
    rng = np.random.default_rng(1)
    a = rng.standard_normal((64, 128)).astype(np.float32)
    b = rng.standard_normal((48, 128)).astype(np.float32)
    qa = oracle.quantize(a, oracle.NVFP4, rotation=oracle.ROT_H16)
    qb = oracle.quantize(b, oracle.NVFP4, rotation=oracle.ROT_H16)
    C, bound = oracle.gemm(qa, qb)
    # the rotation cancels in the contraction: close to the unquantized product
    ref = a.astype(np.float64) @ b.astype(np.float64).T
    rel = np.abs(C - ref).max() / np.abs(ref).max()
    assert rel < 0.2
    assert (bound >= np.abs(C)).all()
