"""Failure detection of the GEMM pipelines and the one-launch quantizer
without a GPU fault.

Every hand-off inside the GEMM kernels (TMA producer -> MMA issuer ->
epilogue, and the double-block GEMM's partial and outer-scale buffers) is an
mbarrier wait bounded by a poll limit.  When a wait runs out, the kernel
raises an abort flag that the other roles see, lets its copies and MMAs in
flight finish, frees TMEM and returns; the host learns of it through
fp4_last_error as FP4_ERR_TIMEOUT.

Here the limit is lowered to one poll (about a microsecond), far below the
time a K = 8192 tile needs, so the first wait of the epilogue runs out.  The
test checks the status, and that the context is still usable: the next call
with the default limit gives the same bits as a call made before the timeout,
and reports FP4_OK.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def operands(fp4, fmt, double_block, M=256, N=256, K=8192, seed=5):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn((M, K), generator=g).to(torch.bfloat16).cuda()
    b = torch.randn((N, K), generator=g).to(torch.bfloat16).cuda()
    kw = dict(fmt=fmt, double_block=double_block, axis=1)
    return fp4.quantize(a, tensor_id=1, **kw), fp4.quantize(b, tensor_id=2, **kw)


# (M, N) = (256, 256) runs on one CTA pair unless pairs are switched off, and
# (512, 256) on two; the pair kernel's leader then also settles the loads
# that only one of the two CTAs issued before it gave up.
@pytest.mark.parametrize("fmt,double_block,out,pairs,M", [
    ("MXFP4", False, "F32", True, 256),
    ("NVFP4", False, "BF16", True, 256),
    ("NVFP4", False, "F32", True, 512),
    ("MXFP4", False, "F32", False, 256),
    ("NVFP4", False, "BF16", False, 256),
    ("NVFP4", True, "BF16", False, 256),
    ("NVFP4", True, "F32", False, 256),
])
def test_gemm_wait_timeout_is_reported_and_recoverable(fp4, fmt, double_block, out, pairs, M):
    qa, qb = operands(fp4, getattr(fp4, "FP4_" + fmt), double_block, M=M)
    out_dtype = getattr(fp4, "FP4_OUT_" + out)
    fp4.fp4_set_gemm_cta_pairs(pairs)
    try:
        before = fp4.gemm(qa, qb, out_dtype)
        assert fp4.fp4_last_error() == fp4.FP4_OK

        fp4.fp4_set_wait_limit(1)
        try:
            fp4.gemm(qa, qb, out_dtype)
            status = fp4.fp4_last_error()
        finally:
            fp4.fp4_set_wait_limit(0)
        assert status == fp4.FP4_ERR_TIMEOUT, fp4.fp4_status_string(status)

        after = fp4.gemm(qa, qb, out_dtype)
    finally:
        fp4.fp4_set_gemm_cta_pairs(True)
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert torch.equal(before.view(torch.int16 if out == "BF16" else torch.int32),
                       after.view(torch.int16 if out == "BF16" else torch.int32))


# The one-launch quantizer (tensor amax pass, grid barrier, quantize pass)
# waits on its shared-memory ring and on the grid barrier; both budgets follow
# the wait limit (16 x and 4 x).  At one poll the barrier runs out long before
# every CTA has finished the amax pass of a 8192 x 4096 tensor.  The kernel
# lets its own bulk copies land before it exits; the next call at the default
# limit must give the bytes a call before the timeout gave.
@pytest.mark.parametrize("fmt,rounding,rotation", [("NVFP4", 0, 1), ("UFP4", 1, 3)])
def test_one_launch_quantizer_wait_timeout_is_reported_and_recoverable(fp4, fmt, rounding, rotation):
    g = torch.Generator().manual_seed(11)
    x = torch.randn((8192, 4096), generator=g).to(torch.bfloat16).cuda()
    kw = dict(fmt=getattr(fp4, "FP4_" + fmt), rounding=rounding, rotation=rotation, axis=1, seed=3, tensor_id=2)
    before = fp4.quantize(x, **kw)
    assert fp4.fp4_last_error() == fp4.FP4_OK

    fp4.fp4_set_wait_limit(1)
    try:
        fp4.quantize(x, **kw)
        status = fp4.fp4_last_error()
    finally:
        fp4.fp4_set_wait_limit(0)
    assert status == fp4.FP4_ERR_TIMEOUT, fp4.fp4_status_string(status)

    after = fp4.quantize(x, **kw)
    assert fp4.fp4_last_error() == fp4.FP4_OK
    for key in ("codes", "tensor_scale"):
        assert torch.equal(before[key].view(torch.uint8), after[key].view(torch.uint8)), key
    n = fp4.fp4_scales_bytes(8192, 4096, kw["fmt"])
    assert torch.equal(before["scales"][:n], after["scales"][:n])


# The both-axes quantizer (column kernel with the row part) runs the same
# bounded ring and grid-barrier waits; at one poll they run out, the call is
# reported, and the next call at the default limit gives the earlier bytes.
def test_both_axes_quantizer_wait_timeout_is_reported_and_recoverable(fp4):
    g = torch.Generator().manual_seed(12)
    x = torch.randn((8192, 4096), generator=g).to(torch.bfloat16).cuda()
    kw = dict(fmt=fp4.FP4_NVFP4, rotation=1, seed=3, rounding_rows=0, tensor_id_rows=1, rounding_cols=1,
              tensor_id_cols=2)
    before = fp4.quantize_both_axes(x, **kw)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK

    fp4.fp4_set_wait_limit(1)
    try:
        fp4.quantize_both_axes(x, **kw)
        status = fp4.fp4_last_error()
    finally:
        fp4.fp4_set_wait_limit(0)
    assert status == fp4.FP4_ERR_TIMEOUT, fp4.fp4_status_string(status)

    after = fp4.quantize_both_axes(x, **kw)
    assert fp4.fp4_last_error() == fp4.FP4_OK
    for b, a in zip(before, after):
        for key in ("codes", "scales", "tensor_scale"):
            assert torch.equal(b[key].view(torch.uint8), a[key].view(torch.uint8)), key
