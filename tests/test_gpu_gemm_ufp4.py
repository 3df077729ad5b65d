"""The UFP4 GEMM ("Ripensare il Bias di Shrinkage nel Pretraining di LLM in
FP4", Metodologia 2: the uniform grid k s, k in [-7, 7], on all three training
GEMMs) against the oracle's float64 GEMM of the exactly dequantized operands,
per element within |C - C64| <= 1e-5 sum_k |a_ik b_jk| (+ half a bf16 ulp for
bf16 output).  The library runs it as an NVFP4 GEMM over the operands' exact
E2M1 parts (fp4_gemm in include/fp4.h); nothing here depends on that.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (assert_quant_equal, assert_within_gemm_bound, gpu_quantize, oracle_quantize,
                    upload_oracle_qtensor)

pytestmark = pytest.mark.gpu
UF = 2


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def rand(M, K, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) * scale).astype(np.float32)
    x[:, rng.choice(K, 2, replace=False)] *= 30.0
    return torch.from_numpy(x)


@pytest.mark.parametrize("out_bf16", [False, True])
@pytest.mark.parametrize("shape", [(128, 128, 256), (256, 384, 512), (128, 256, 128), (256, 128, 384),
                                   (384, 512, 1152), (128, 256, 4096), (5120, 1024, 256)])
def test_ufp4_gemm_on_oracle_operands(fp4, shape, out_bf16):
    M, N, K = shape
    a, b = rand(M, K, M + K + 1), rand(N, K, N + 3 * K, 0.1)
    qa = oracle_quantize(a, fmt=UF, rotation=1)
    qb = oracle_quantize(b, fmt=UF, rotation=1, rounding=1, seed=2, tensor_id=7)
    C64, bound = oracle.gemm(qa, qb)
    C = fp4.gemm(upload_oracle_qtensor(fp4, qa), upload_oracle_qtensor(fp4, qb),
                 fp4.FP4_OUT_BF16 if out_bf16 else fp4.FP4_OUT_F32)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert_within_gemm_bound(C.float().cpu().numpy(), C64, bound, out_bf16, what=str((shape, out_bf16)))


def test_ufp4_gemm_every_code_pair(fp4):
    # every pair of codes (sign and k) meets in some product, with scales that
    # make each block's weight distinct
    rng = np.random.default_rng(5)
    M, N, K = 128, 128, 256
    ca = np.stack([rng.permutation(np.tile(np.arange(16, dtype=np.uint8), K // 16)) for _ in range(M)])
    cb = np.stack([rng.permutation(np.tile(np.arange(16, dtype=np.uint8), K // 16)) for _ in range(N)])
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    qa = dict(codes=pack(ca), scales=rng.integers(1, 0x7F, (M, K // 16)).astype(np.uint8), outer=None,
              tensor_scale=np.float32(0.37), K=K, format=UF, double_block=False)
    qb = dict(codes=pack(cb), scales=rng.integers(1, 0x7F, (N, K // 16)).astype(np.uint8), outer=None,
              tensor_scale=np.float32(1.9), K=K, format=UF, double_block=False)
    C64, bound = oracle.gemm(qa, qb)
    C = fp4.gemm(upload_oracle_qtensor(fp4, qa), upload_oracle_qtensor(fp4, qb), fp4.FP4_OUT_F32)
    torch.cuda.synchronize()
    assert_within_gemm_bound(C.cpu().numpy(), C64, bound, False, what="every code pair")


@pytest.mark.parametrize("rot", [0, 1, 3])
def test_ufp4_quantize_then_gemm(fp4, rot):
    """The whole UFP4 path: quantize both operands on the GPU, then the GEMM."""
    a, b = rand(384, 1024, 11 + rot), rand(256, 1024, 12 + rot, 0.05)
    kw = dict(fmt=UF, rotation=rot, seed=4)
    ga = gpu_quantize(fp4, a.cuda(), tensor_id=1, **kw)
    gb = gpu_quantize(fp4, b.to(torch.bfloat16).cuda(), tensor_id=2, rounding=1, **kw)
    oa = oracle_quantize(a, tensor_id=1, **kw)
    ob = oracle_quantize(b.to(torch.bfloat16), tensor_id=2, rounding=1, **kw)
    assert_quant_equal(ga, oa)
    assert_quant_equal(gb, ob)
    C = fp4.gemm(ga["raw"], gb["raw"], fp4.FP4_OUT_BF16)
    torch.cuda.synchronize()
    C64, bound = oracle.gemm(oa, ob)
    assert_within_gemm_bound(C.float().cpu().numpy(), C64, bound, True)
