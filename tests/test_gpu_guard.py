"""Guard bytes around every output: each output buffer sits inside a larger
allocation filled with a canary pattern, at a 16-byte aligned offset, and
after the call every byte outside the output (and outside the valid part of
the tiled scale layout's padding) must still hold the canary.  Covers the row
and column quantizers (ragged shapes, every format), the one-launch amax path,
the re-quantize, and both GEMMs with ldc > N."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

CANARY = 0xA5
PAD = 256


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def guarded(nbytes, dev="cuda"):
    """(whole buffer, view of nbytes at offset PAD) filled with the canary."""
    whole = torch.full((nbytes + 2 * PAD,), CANARY, dtype=torch.uint8, device=dev)
    return whole, whole[PAD:PAD + nbytes]


def assert_guards(whole, nbytes, what):
    w = whole.cpu().numpy()
    assert (w[:PAD] == CANARY).all(), what + ": bytes before the buffer were written"
    assert (w[PAD + nbytes:] == CANARY).all(), what + ": bytes after the buffer were written"


def guarded_qtensor(fp4, L, K, fmt, db):
    nb_codes = L * K // 2
    nb_scales = max(fp4.fp4_scales_bytes(L, K, fmt), 16)
    nb_outer = L * max(K // 128, 1) * 4
    gc, codes = guarded(nb_codes)
    gs, scales = guarded(nb_scales)
    go, outer = guarded(nb_outer)
    gt, ts = guarded(4)
    q = dict(codes=codes.view(L, K // 2), scales=scales, outer=outer.view(torch.float32).view(L, -1) if db else None,
             tensor_scale=ts.view(torch.float32), lines=L, K=K, format=fmt, double_block=db)
    guards = [(gc, nb_codes, "codes"), (gs, nb_scales, "scales"), (gt, 4, "tensor scale")]
    if db:
        guards.append((go, nb_outer, "outer"))
    return q, guards


@pytest.mark.parametrize("axis", [1, 0])
@pytest.mark.parametrize("fmt,db,rounding,rot", [(0, False, 1, 4), (1, False, 0, 1), (1, True, 1, 0), (2, False, 0, 3)])
def test_quantize_writes_only_its_outputs(fp4, axis, fmt, db, rounding, rot):
    R, C = (272, 384) if axis == 1 else (384, 272)      # 272 lines: a ragged 128-line group
    x = torch.randn((R, C), generator=torch.Generator().manual_seed(R + fmt)).to(torch.bfloat16).cuda()
    L, K = (R, C) if axis == 1 else (C, R)
    q, guards = guarded_qtensor(fp4, L, K, fmt, db)
    fp4.quantize(x, fmt, rounding, rot, axis=axis, double_block=db, seed=1, tensor_id=2, out=q)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    for whole, n, what in guards:
        assert_guards(whole, n, "%s axis %d fmt %d" % (what, axis, fmt))


def test_requantize_writes_only_its_outputs(fp4):
    x = torch.randn((384, 272), generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    src = fp4.quantize(x, 1, 0, 0, axis=1)
    q, guards = guarded_qtensor(fp4, 272, 384, 1, True)
    fp4.requantize(src, 1, 1, double_block=True, seed=2, tensor_id=1, out=q)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    for whole, n, what in guards:
        assert_guards(whole, n, "requantize " + what)


@pytest.mark.parametrize("K", [512, 384])              # 384: the last K stage is half a stage
@pytest.mark.parametrize("fmt,db", [(0, False), (1, False), (1, True)])
@pytest.mark.parametrize("N,ldc", [(384, 392), (512, 520)])   # 512: CTA-pair tiles (not for the double block)
def test_gemm_writes_only_c_rows_and_columns(fp4, fmt, db, K, N, ldc):
    M = 256                                              # ldc > N: 8 padding columns per row
    g = torch.Generator().manual_seed(fmt)
    a = torch.randn((M, K), generator=g).to(torch.bfloat16).cuda()
    b = torch.randn((N, K), generator=g).to(torch.bfloat16).cuda()
    qa = fp4.quantize(a, fmt, double_block=db)
    qb = fp4.quantize(b, fmt, double_block=db)
    nbytes = M * ldc * 2
    whole, cbuf = guarded(nbytes)
    out = cbuf.view(torch.bfloat16).view(M, ldc)[:, :N]
    fp4.gemm(qa, qb, fp4.FP4_OUT_BF16, out=out)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert_guards(whole, nbytes, "C")
    pad = cbuf.view(M, ldc * 2)[:, 2 * N:].cpu().numpy()
    assert (pad == CANARY).all(), "the padding columns between rows of C were written"
