"""GEMM parity: the tcgen05 block-scaled FP4 GEMM (through the C ABI) against
the oracle's float64 GEMM of the exactly dequantized operands, per element
within |C - C64| <= 1e-5 * sum_k |a_ik b_jk| (plus half a bf16 ulp of the
result for bf16 output).

Operands: first the oracle's own quantized tensors uploaded to the GPU (the
GEMM alone), then the whole path (GPU quantizer -> GPU GEMM against oracle
quantizer -> oracle GEMM), at small sizes in full and at the full
Llama-3.1-8B-shaped sizes on sampled rows and columns.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (assert_quant_equal, assert_within_gemm_bound, gpu_quantize, oracle_quantize,
                    sample_lines, upload_oracle_qtensor)
from fp4_block_scaled_h16_b200 import workloads

pytestmark = pytest.mark.gpu
MX, NV = 0, 1


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def rand(M, K, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) * scale).astype(np.float32)
    x[:, rng.choice(K, 2, replace=False)] *= 30.0
    return torch.from_numpy(x)


@pytest.fixture(params=[True, False], ids=["pairs", "single"])
def cta_pairs(fp4, request):
    """Runs the test with 256 x 256 tiles on CTA pairs where M and N allow it
    (the default), then with single-CTA 128 x 256 tiles only."""
    fp4.fp4_set_gemm_cta_pairs(request.param)
    yield request.param
    fp4.fp4_set_gemm_cta_pairs(True)


@pytest.mark.parametrize("out_bf16", [False, True])
@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("shape", [(128, 128, 256), (256, 384, 512), (384, 256, 1024), (128, 512, 2304),
                                   (128, 256, 128), (256, 128, 384), (384, 512, 1152),
                                   (256, 256, 256), (512, 768, 1152), (256, 512, 128), (768, 256, 2048)])
def test_gemm_on_oracle_operands(fp4, fmt, out_bf16, shape, cta_pairs):
    M, N, K = shape
    a, b = rand(M, K, M + K + fmt), rand(N, K, N + 3 * K + fmt, 0.1)
    qa = oracle_quantize(a, fmt=fmt, rotation=1)
    qb = oracle_quantize(b, fmt=fmt, rotation=1)
    C64, bound = oracle.gemm(qa, qb)
    ta, tb = upload_oracle_qtensor(fp4, qa), upload_oracle_qtensor(fp4, qb)
    C = fp4.gemm(ta, tb, fp4.FP4_OUT_BF16 if out_bf16 else fp4.FP4_OUT_F32)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert_within_gemm_bound(C.float().cpu().numpy(), C64, bound, out_bf16, what=str((fmt, shape, out_bf16)))


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("out_bf16", [True, False])
@pytest.mark.parametrize("shape", [(5120, 1024, 256), (2560, 2048, 512), (5120, 1024, 384), (4096, 5120, 256)])
def test_gemm_with_more_tiles_than_sms_on_oracle_operands(fp4, fmt, shape, out_bf16, cta_pairs):
    # single CTAs: more 128x256 tiles than SMs (160 tiles on 148 SMs: a
    # second, nearly empty wave of persistent tiles, run as 128-column halves;
    # K = 384 ends on a half stage).  CTA pairs: 80 256x256 tiles on 74 pairs,
    # a second wave of 6, run as 256x128 halves; 4096 x 5120: 320 pair tiles,
    # a last wave of 24 as 48 halves (640 single tiles, a last wave of 48 as
    # 96 halves).  Every element against the oracle.
    M, N, K = shape
    a, b = rand(M, K, M + fmt), rand(N, K, N + 7 + fmt, 0.1)
    qa = oracle_quantize(a, fmt=fmt)
    qb = oracle_quantize(b, fmt=fmt)
    C64, bound = oracle.gemm(qa, qb)
    C = fp4.gemm(upload_oracle_qtensor(fp4, qa), upload_oracle_qtensor(fp4, qb),
                 fp4.FP4_OUT_BF16 if out_bf16 else fp4.FP4_OUT_F32)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert_within_gemm_bound(C.float().cpu().numpy(), C64, bound, out_bf16, what=str((fmt, shape, out_bf16)))


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("shape", [(512, 512, 1024), (2048, 1536, 640), (5120, 1024, 384)])
def test_pair_and_single_cta_tiles_give_the_same_bits(fp4, fmt, shape):
    """The pair MMA (M = 256 over two SMs) and the single-CTA MMA (M = 128)
    take the same 64-element K slices in the same order for every output, so
    the two paths agree bit for bit; both stay within the oracle's bound."""
    M, N, K = shape
    a, b = rand(M, K, 3 * M + fmt), rand(N, K, 5 * N + fmt, 0.1)
    qa, qb = oracle_quantize(a, fmt=fmt, rotation=1), oracle_quantize(b, fmt=fmt, rotation=1)
    ta, tb = upload_oracle_qtensor(fp4, qa), upload_oracle_qtensor(fp4, qb)
    out = {}
    try:
        for pairs in (True, False):
            fp4.fp4_set_gemm_cta_pairs(pairs)
            out[pairs] = fp4.gemm(ta, tb, fp4.FP4_OUT_F32)
            torch.cuda.synchronize()
            assert fp4.fp4_last_error() == fp4.FP4_OK
    finally:
        fp4.fp4_set_gemm_cta_pairs(True)
    C64, bound = oracle.gemm(qa, qb)
    for pairs in (True, False):
        assert_within_gemm_bound(out[pairs].cpu().numpy(), C64, bound, False, what=str((fmt, shape, pairs)))
    assert torch.equal(out[True].view(torch.int32), out[False].view(torch.int32))


@pytest.mark.parametrize("M", [128, 256])              # 256: CTA-pair tiles, C written by tiled stores
def test_gemm_ldc_larger_than_n(fp4, M):
    a, b = rand(M, 512, 1), rand(256, 512, 2)
    qa, qb = oracle_quantize(a, fmt=NV), oracle_quantize(b, fmt=NV)
    C64, bound = oracle.gemm(qa, qb)
    out = torch.full((M, 264), 7.0, dtype=torch.float32, device="cuda")
    fp4.gemm(upload_oracle_qtensor(fp4, qa), upload_oracle_qtensor(fp4, qb), fp4.FP4_OUT_F32,
             out=out[:, :256])
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    assert (o[:, 256:] == 7.0).all()
    assert_within_gemm_bound(o[:, :256], C64, bound, False)


def test_gemm_zero_and_extreme_scales(fp4):
    a = torch.zeros((128, 512))
    a[3, :] = 1e30
    a[5, :] = 1e-30
    b = rand(128, 512, 9)
    for fmt in (MX, NV):
        qa, qb = oracle_quantize(a, fmt=fmt), oracle_quantize(b, fmt=fmt)
        C64, bound = oracle.gemm(qa, qb)
        C = fp4.gemm(upload_oracle_qtensor(fp4, qa), upload_oracle_qtensor(fp4, qb), fp4.FP4_OUT_F32)
        torch.cuda.synchronize()
        assert_within_gemm_bound(C.cpu().numpy(), C64, bound, False)


def test_tiny_mxfp4_end_to_end(fp4):
    """A fp32 256x512 (axis 1) times B fp32 512x256 (axis 0): C = A B, fp32 out."""
    d = workloads.tiny_mxfp4()
    ga = gpu_quantize(fp4, d["A"].cuda(), fmt=MX, axis=1)
    gb = gpu_quantize(fp4, d["B"].cuda(), fmt=MX, axis=0)
    oa, ob = oracle_quantize(d["A"], fmt=MX, axis=1), oracle_quantize(d["B"], fmt=MX, axis=0)
    assert_quant_equal(ga, oa)
    assert_quant_equal(gb, ob)
    C = fp4.gemm(ga["raw"], gb["raw"], fp4.FP4_OUT_F32)
    torch.cuda.synchronize()
    C64, bound = oracle.gemm(oa, ob)
    assert_within_gemm_bound(C.cpu().numpy(), C64, bound, False, what="tiny")
    # the quantized product is close to the exact one
    ref = d["A"].double().numpy() @ d["B"].double().numpy()
    assert np.abs(C.cpu().numpy() - ref).max() < 0.25 * np.abs(ref).max()


def sampled_gemm_check(fp4, qa_dev, qb_dev, x_a, x_b, kw_a, kw_b, out_bf16, n, seed):
    C = fp4.gemm(qa_dev, qb_dev, fp4.FP4_OUT_BF16 if out_bf16 else fp4.FP4_OUT_F32)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    rows = sample_lines(qa_dev["lines"], n, seed)
    cols = sample_lines(qb_dev["lines"], n, seed + 1)
    oa = oracle_quantize(x_a, lines=rows, **kw_a)
    ob = oracle_quantize(x_b, lines=cols, **kw_b)
    C64, bound = oracle.gemm(oa, ob)
    sub = C.float()[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].cpu().numpy()
    return assert_within_gemm_bound(sub, C64, bound, out_bf16)


def test_full_nvfp4_fprop_qkv(fp4):
    """Y = X W^T, X 8192x4096, W 6144x4096, NVFP4 + H16, bf16 out 8192x6144."""
    d = workloads.nvfp4_fprop_qkv()
    kw = dict(fmt=NV, rounding=0, rotation=1, axis=1)
    qx = fp4.quantize(d["X"].cuda(), **kw)
    qw = fp4.quantize(d["W"].cuda(), **kw)
    sampled_gemm_check(fp4, qx, qw, d["X"], d["W"], kw, kw, True, 128, 0)


def test_full_mxfp4_wgrad_down(fp4):
    """dW = dY^T H: both quantized along the 8192 tokens, random-sign H32, SR; fp32 out 4096x14336."""
    d = workloads.mxfp4_wgrad_down()
    ka = dict(fmt=MX, rounding=1, rotation=4, axis=0, seed=0, tensor_id=1)
    kb = dict(fmt=MX, rounding=1, rotation=4, axis=0, seed=0, tensor_id=2)
    qa = fp4.quantize(d["dY"].cuda(), **ka)
    qb = fp4.quantize(d["H"].cuda(), **kb)
    sampled_gemm_check(fp4, qa, qb, d["dY"], d["H"], ka, kb, False, 96, 1)


@pytest.mark.parametrize("out_bf16", [False, True])
@pytest.mark.parametrize("shape", [(128, 128, 256), (256, 384, 512), (128, 256, 2048), (384, 128, 8192),
                                   (128, 128, 128), (256, 128, 384), (128, 256, 1152), (128, 128, 8064),
                                   (128, 128, 8320), (256, 128, 16384), (128, 256, 24704)])
def test_double_block_gemm_on_oracle_operands(fp4, out_bf16, shape):
    """C = sum over 128-K chunks of s_oA * s_oB * (block-scaled partial).  K
    past 8192 takes B's outer scales in several staged groups of 64 chunks
    (8320: 64 + 1, 16384: 64 + 64, 24704: 3 x 64 + 1)."""
    M, N, K = shape
    a, b = rand(M, K, M + K), rand(N, K, 7 * N + K, 0.1)
    # chunk magnitudes that vary along K on both operands, so every chunk's
    # outer scales matter (and a group taken for the wrong chunks shows)
    a = a * torch.from_numpy(np.repeat(np.exp2(np.random.default_rng(1).integers(-6, 6, K // 128)), 128)).float()
    b = b * torch.from_numpy(np.repeat(np.exp2(np.random.default_rng(2).integers(-6, 6, K // 128)), 128)).float()
    qa = oracle_quantize(a, fmt=NV, double_block=True, rounding=1, seed=3, tensor_id=1)
    qb = oracle_quantize(b, fmt=NV, double_block=True, rounding=1, seed=3, tensor_id=2)
    C64, bound = oracle.gemm(qa, qb)
    C = fp4.gemm(upload_oracle_qtensor(fp4, qa), upload_oracle_qtensor(fp4, qb),
                 fp4.FP4_OUT_BF16 if out_bf16 else fp4.FP4_OUT_F32)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert_within_gemm_bound(C.float().cpu().numpy(), C64, bound, out_bf16, what="db %s" % (shape,))


def test_full_nvfp4_dgrad_double_block(fp4):
    """dH = dY Wd: dY 8192x4096 (axis 1), Wd 4096x14336 quantized along its
    transposed axis (axis 0), double block, SR; bf16 out 8192x14336."""
    d = workloads.nvfp4_dgrad_down()
    ka = dict(fmt=NV, rounding=1, rotation=0, axis=1, double_block=True, seed=0, tensor_id=1)
    kb = dict(fmt=NV, rounding=1, rotation=0, axis=0, double_block=True, seed=0, tensor_id=2)
    qa = fp4.quantize(d["dY"].cuda(), **ka)
    qb = fp4.quantize(d["Wd"].cuda(), **kb)
    sampled_gemm_check(fp4, qa, qb, d["dY"], d["Wd"], ka, kb, True, 96, 2)


def test_double_block_gemm_long_k_whole_path(fp4):
    """The double-block GEMM at K = 28672 (the gate+up Dgrad's contraction) on
    GPU-quantized operands, sampled rows and columns against the oracle."""
    M, N, K = 256, 512, 28672
    a, b = rand(M, K, 11), rand(N, K, 12, 0.1)
    ka = dict(fmt=NV, rounding=1, rotation=0, axis=1, double_block=True, seed=0, tensor_id=1)
    kb = dict(fmt=NV, rounding=1, rotation=0, axis=1, double_block=True, seed=0, tensor_id=2)
    qa = fp4.quantize(a.bfloat16().cuda(), **ka)
    qb = fp4.quantize(b.bfloat16().cuda(), **kb)
    sampled_gemm_check(fp4, qa, qb, a.bfloat16(), b.bfloat16(), ka, kb, True, 64, 3)
