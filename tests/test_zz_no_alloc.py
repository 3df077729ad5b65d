"""fp4_quantize_noalloc -- the entry point for callers that cannot allocate
device memory (a plug-in whose host framework owns every device allocation, a
loop that may not touch the allocator): its scratch is a static array inside
libfp4.so.  It must give exactly what fp4_quantize with a caller workspace
gives, call after call, and both must agree with the CPU oracle.

Collected last on purpose: the static scratch keeps the previous call's
contents, so this must hold both in a fresh process and after every other
test has used the library.
"""
import numpy as np
import pytest
import torch

from parity import assert_quant_equal, oracle_quantize, untile

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def inputs(seed, R, C, scale):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((R, C), generator=g) * scale
    x[:, 7] *= 40.0
    return x.to(torch.bfloat16).cuda()


def via_workspace(fp4, x, fmt, rounding, rotation, axis, seed, tid):
    q = fp4.quantize(x, fmt, rounding, rotation, axis=axis, seed=seed, tensor_id=tid)
    torch.cuda.synchronize()
    return q


def via_noalloc(fp4, x, fmt, rounding, rotation, axis, seed, tid):
    R, C = x.shape
    L, K = (R, C) if axis == 1 else (C, R)
    q = fp4.alloc_qtensor(L, K, fmt, device=x.device)
    fp4.fp4_quantize_noalloc(x, fp4.FP4_IN_BF16, R, C, C, fmt, rounding, rotation, axis, seed, tid,
                             q["codes"], q["scales"], q["tensor_scale"])
    torch.cuda.synchronize()
    return q


def same(fp4, a, b):
    L, K = a["lines"], a["K"]
    nb = K // 16
    assert torch.equal(a["codes"], b["codes"])
    assert torch.equal(a["tensor_scale"], b["tensor_scale"])
    # compare the written scale bytes (the tiled padding is never written)
    idx = torch.from_numpy(np.array([[((l // 128) * ((nb + 3) // 4) + j // 4) * 512 + (l % 32) * 16
                                       + ((l % 128) // 32) * 4 + j % 4 for j in range(nb)]
                                     for l in range(L)]).ravel()).cuda()
    assert torch.equal(a["scales"][idx], b["scales"][idx])


@pytest.mark.parametrize("fmt,rounding,rotation,axis", [(1, 0, 1, 1), (2, 1, 4, 0), (1, 1, 3, 0)])
def test_noalloc_matches_workspace_path_two_calls(fp4, fmt, rounding, rotation, axis):
    # the second input has a much smaller amax than the first: an uncleared
    # slot from the first call would give it the wrong tensor scale
    for i, scale in enumerate((3.0, 0.01)):
        x = inputs(100 * fmt + i, 384, 512, scale)
        a = via_workspace(fp4, x, fmt, rounding, rotation, axis, 11, 5 + i)
        b = via_noalloc(fp4, x, fmt, rounding, rotation, axis, 11, 5 + i)
        same(fp4, a, b)
        # and the static-scratch result is the oracle's, bit for bit
        o = oracle_quantize(x.cpu(), fmt=fmt, rounding=rounding, rotation=rotation, axis=axis, seed=11,
                            tensor_id=5 + i)
        g = dict(codes=b["codes"].cpu().numpy(),
                 scales=untile(b["scales"].cpu().numpy(), b["lines"], b["K"], fmt),
                 outer=None, tensor_scale=float(b["tensor_scale"].cpu()[0]))
        assert_quant_equal(g, o, what="noalloc call %d" % i)


def test_noalloc_rejects_mxfp4_and_bad_args(fp4):
    x = inputs(1, 128, 256, 1.0)
    q = fp4.alloc_qtensor(128, 256, fp4.FP4_NVFP4, device=x.device)
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.fp4_quantize_noalloc(x, fp4.FP4_IN_BF16, 128, 256, 256, fp4.FP4_MXFP4, 0, 0, 1, 0, 0,
                                 q["codes"], q["scales"], q["tensor_scale"])
    assert e.value.status == fp4.FP4_ERR_UNSUPPORTED
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.fp4_quantize_noalloc(x, fp4.FP4_IN_BF16, 128, 248, 256, fp4.FP4_NVFP4, 0, 0, 1, 0, 0,
                                 q["codes"], q["scales"], q["tensor_scale"])
    assert e.value.status == fp4.FP4_ERR_UNSUPPORTED_SHAPE
