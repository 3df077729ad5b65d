"""MXNorm fused with the FP4 cast (fp4_mxnorm_quantize, "MXNorm: Reusing MXFP
block scales for efficient tensor normalisation", 2. Metodologia) against the
oracle, bit for bit: rho per row, codes, scales and the tensor scale.

Shapes: ragged row counts; block counts per row that are not powers of two
(the pairwise sum's zero padding); the FFN width 14336; a row pitch wider than
the row; special rows (all zero, subnormal, one huge outlier, signed zeros);
the layer's 8192 x 4096 activation at full size on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_quant_equal, oracle_input, sample_lines, untile, untile_lines
from fp4_block_scaled_h16_b200 import workloads

pytestmark = pytest.mark.gpu
MX, NV, UF = 0, 1, 2


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def c_of(p, fmt):
    return float(np.float32(oracle.mxnorm_constant(p, 32 if fmt == MX else 16)))


def compare(fp4, q, o, lines=None, what=""):
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    L, K, fmt = q["lines"], q["K"], q["format"]
    rho = q["rho"].cpu().numpy()[:L]
    if lines is None:
        g = dict(codes=q["codes"].cpu().numpy(), scales=untile(q["scales"].cpu().numpy(), L, K, fmt), outer=None,
                 tensor_scale=float(q["tensor_scale"].cpu()[0]))
        assert (rho.view(np.uint32) == o["rho"].view(np.uint32)).all(), (what, rho[:4], o["rho"][:4])
        assert_quant_equal(g, o, what=what)
    else:
        idx = torch.from_numpy(lines).cuda()
        g = dict(codes=q["codes"][idx].cpu().numpy(), scales=untile_lines(q["scales"].cpu().numpy(), lines, K, fmt),
                 outer=None, tensor_scale=float(q["tensor_scale"].cpu()[0]))
        assert (rho.view(np.uint32) == o["rho"].view(np.uint32)).all(), what
        assert_quant_equal(g, o, lines=np.arange(len(lines)), what=what)


def make(R, ld, dtype, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, ld)).astype(np.float32) * np.exp2(rng.integers(-6, 6, (R, 1))).astype(np.float32)
    x[:, rng.choice(ld, 2, replace=False)] *= 40.0
    t = torch.from_numpy(x)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rounding", [0, 1])
@pytest.mark.parametrize("p", [1, 2])
@pytest.mark.parametrize("fmt", [MX, NV, UF])
# bf16 rows of 256 .. 4096 columns (a multiple of 256) run one warp per row
# (11 and 5 chunks of 256: chunk sums padded to a power of two; a row pitch
# wider than the row); the other shapes and f32 take the CTA-per-row kernel
@pytest.mark.parametrize("shape", [(37, 4096, 4096), (5, 14336, 14336), (130, 96, 128), (64, 4128, 4160),
                                   (300, 2816, 2816), (70, 256, 264), (9, 1280, 1280)])
def test_mxnorm_matches_oracle(fp4, fmt, p, rounding, dtype, shape):
    R, C, ld = shape
    if C % (32 if fmt == MX else 16):
        pytest.skip("block does not divide the row")
    full = make(R, ld, dtype, seed=R + C + 10 * fmt + p)
    c = c_of(p, fmt)
    q = fp4.mxnorm_quantize(full.cuda()[:, :C], fmt, p, c, rounding=rounding, seed=5, tensor_id=9)
    o = oracle.mxnorm(oracle_input(full), fmt, p, c, rounding=rounding, seed=5, tensor_id=9, C=C)
    compare(fp4, q, o, what=str((fmt, p, rounding, dtype, shape)))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("p", [1, 2])
def test_mxnorm_special_rows(fp4, fmt, p, dtype):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((8, 512)).astype(np.float32)
    x[0] = 0.0                       # all zero: rho = 1
    x[1] = -0.0
    x[1, ::7] = 1.0                  # signed zeros among nonzero values
    x[2] = np.float32(2.0 ** -149)   # subnormal row: rho saturates
    x[3] = 1e-3
    x[3, 100] = 3e4                  # one huge outlier
    x[4] = 1e30
    x[5, ::2] = 0.0
    c = c_of(p, fmt)
    xt = torch.from_numpy(x)
    if dtype == "bf16":
        xt = xt.to(torch.bfloat16)       # the subnormal row becomes zeros; 512 columns: the warp-per-row kernel
    q = fp4.mxnorm_quantize(xt.cuda(), fmt, p, c)
    o = oracle.mxnorm(oracle_input(xt), fmt, p, c)
    compare(fp4, q, o, what="special %s" % ((fmt, p, dtype),))
    assert o["rho"][0] == 1.0


@pytest.mark.parametrize("fmt", [MX, NV])
def test_mxnorm_full_activation(fp4, fmt):
    """The layer's QKV input, 8192 x 4096 bf16 with outlier channels, p = 2."""
    d = workloads.layer_linear("qkv")
    c = c_of(2, fmt)
    q = fp4.mxnorm_quantize(d["X"].cuda(), fmt, 2, c)
    lines = sample_lines(8192, 64, 3)
    o = oracle.mxnorm(oracle_input(d["X"]), fmt, 2, c, lines=lines)
    compare(fp4, q, o, lines=lines, what="full %d" % fmt)


def test_mxnorm_rejects(fp4):
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    q = fp4.alloc_qtensor(4, 64, MX, device="cuda")
    rho = torch.empty(4, device="cuda")
    for kw, status in [(dict(p=3), fp4.FP4_ERR_INVALID_ARG), (dict(c=0.0), fp4.FP4_ERR_INVALID_ARG),
                       (dict(c=float("inf")), fp4.FP4_ERR_INVALID_ARG), (dict(cols=48), fp4.FP4_ERR_UNSUPPORTED_SHAPE)]:
        a = dict(p=2, c=2.0, cols=64)
        a.update(kw)
        with pytest.raises(fp4.Fp4Error) as e:
            fp4.fp4_mxnorm_quantize(x, fp4.FP4_IN_BF16, 4, a["cols"], 64, MX, 0, a["p"], a["c"], 0, 0, q["codes"],
                                    q["scales"], q["tensor_scale"], rho, None, 0)
        assert e.value.status == status
