"""fp4_rotate -- the rotation alone, the unfused form the pages time against
the fused quantizer ("Ripensare il Bias di Shrinkage nel Pretraining di LLM in
FP4", Efficienza) -- against the oracle's rotation of every aligned block,
bit for bit (a bf16 output is the binary32 result rounded to nearest even).

In binary32 the rotation is exactly the quantizer's step 2, so rotating and
then quantizing without rotation must give the fused quantizer's codes.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_quant_equal, gpu_quantize, oracle_input

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def oracle_rotate_rows(x: np.ndarray, n: int, signs) -> np.ndarray:
    """binary32 rotation of every aligned n-block of every row, by the oracle."""
    y = np.empty_like(x, dtype=np.float32)
    for r in range(x.shape[0]):
        for b in range(0, x.shape[1], n):
            y[r, b:b + n] = oracle.rotate_block(x[r, b:b + n], signs)
    return y


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rot,n", [(1, 16), (2, 32), (3, 16), (4, 32)])
def test_rotate_matches_oracle(fp4, dtype, rot, n):
    R, C, ld = 77, 320, 352
    g = torch.Generator().manual_seed(rot + 10 * (dtype == torch.bfloat16))
    full = (torch.randn((R, ld), generator=g) * 3.0).to(dtype)
    full[:, 5] *= 1000.0
    x = full[:, :C]
    y = fp4.rotate(full.cuda()[:, :C], rot, seed=0x5EED)
    torch.cuda.synchronize()
    signs = oracle.rht_signs(0x5EED, n) if rot in (3, 4) else None
    want = oracle_rotate_rows(x.float().numpy(), n, signs)
    want_t = torch.from_numpy(want).to(dtype)          # round to nearest even for bf16
    assert torch.equal(y.cpu().view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                       want_t.view(torch.int16 if dtype == torch.bfloat16 else torch.int32))


@pytest.mark.parametrize("fmt,rounding,rot", [(1, 0, 1), (2, 1, 4), (0, 0, 2)])
def test_rotate_then_quantize_equals_fused_in_f32(fp4, fmt, rounding, rot):
    g = torch.Generator().manual_seed(fmt + rot)
    x = (torch.randn((200, 512), generator=g)).cuda()
    kw = dict(fmt=fmt, rounding=rounding, axis=1, seed=9, tensor_id=4)
    fused = gpu_quantize(fp4, x, rotation=rot, **kw)
    unfused = gpu_quantize(fp4, fp4.rotate(x, rot, seed=9), rotation=0, **kw)
    o = oracle.quantize(oracle_input(x.cpu()), fmt, rounding=rounding, rotation=rot, axis=1, seed=9, tensor_id=4)
    assert_quant_equal(fused, o, what="fused")
    assert_quant_equal(unfused, o, what="rotate, then quantize")


def test_rotate_rejects_unsupported(fp4):
    x = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    y = torch.empty_like(x)
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.fp4_rotate(x, fp4.FP4_IN_BF16, 16, 64, 64, fp4.FP4_ROT_H16, 0, 0, y, 64)
    assert e.value.status == fp4.FP4_ERR_UNSUPPORTED
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.fp4_rotate(x, fp4.FP4_IN_BF16, 16, 64, 64, fp4.FP4_ROT_NONE, 1, 0, y, 64)
    assert e.value.status == fp4.FP4_ERR_INVALID_ARG
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.fp4_rotate(x, fp4.FP4_IN_BF16, 16, 48, 64, fp4.FP4_ROT_H32, 1, 0, y, 64)
    assert e.value.status == fp4.FP4_ERR_UNSUPPORTED_SHAPE
