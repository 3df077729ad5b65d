"""Parity of fp4_requantize (the CUDA path, through the C ABI) with the oracle:
X^, the dequantized forward operand, re-quantized along the transposed axis
("TetraJet-v2" 2.A).  The source tensors are the oracle's own quantizations,
uploaded as they are; codes, scales, outer scales and the tensor scale must
match bit for bit.  Shapes include a partial 64-column tile and a partial
128-row tile.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_quant_equal, untile, upload_oracle_qtensor

pytestmark = pytest.mark.gpu

MX, NV, UF = 0, 1, 2


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def source(n, K, fmt, db, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((n, K)) * 0.02).astype(np.float32)
    x[:, rng.choice(K, 2, replace=False)] *= 40.0
    x[rng.choice(n, 2, replace=False), :] *= 1e-3
    return oracle.quantize(x, fmt, double_block=db)


def gpu_requantize(fp4, q_dev, **kw):
    r = fp4.requantize(q_dev, **kw)
    torch.cuda.synchronize()
    L, K, fmt = r["lines"], r["K"], r["format"]
    return dict(codes=r["codes"].cpu().numpy(), scales=untile(r["scales"].cpu().numpy(), L, K, fmt),
                outer=r["outer"].cpu().numpy() if r["outer"] is not None else None,
                tensor_scale=float(r["tensor_scale"].cpu()[0]))


SOURCES = [(MX, False), (NV, False), (NV, True), (UF, False)]
TARGETS = [  # fmt, double block, rounding, rotation
    (MX, False, 0, 0), (MX, False, 1, 4), (NV, False, 0, 1), (NV, False, 1, 0),
    (NV, True, 1, 0), (NV, True, 0, 2), (UF, False, 1, 3), (UF, False, 0, 1),
]


@pytest.mark.parametrize("src", SOURCES)
@pytest.mark.parametrize("tgt", TARGETS)
def test_requantize_matches_oracle(fp4, src, tgt):
    sfmt, sdb = src
    fmt, db, rounding, rot = tgt
    n = 384 if db else 288                  # a partial 128-row tile unless double block
    K = 256 if sdb else 160                 # a partial 64-column tile unless the source is double block
    q = source(n, K, sfmt, sdb, seed=n + K + sfmt)
    kw = dict(fmt=fmt, rounding=rounding, rotation=rot, double_block=db, seed=5, tensor_id=9)
    g = gpu_requantize(fp4, upload_oracle_qtensor(fp4, q), **kw)
    o = oracle.requantize(q, **kw)
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert_quant_equal(g, o, what="requantize %s -> %s" % (src, tgt))


def test_requantize_given_amax_and_special_values(fp4):
    # zeros, signed zeros and tiny values in the source, and a caller-given amax
    x = np.zeros((256, 128), np.float32)
    x[1, :] = -0.0
    x[2, 3] = 5.0
    x[3, :] = 1e-38
    x[4:, :] = np.random.default_rng(1).standard_normal((252, 128)).astype(np.float32)
    q = oracle.quantize(x, NV)
    xhat = oracle.dequantize32(q)
    amax = float(np.abs(xhat).max())
    kw = dict(fmt=NV, rounding=1, rotation=0, seed=2, tensor_id=4)
    ta = torch.tensor([amax], dtype=torch.float32, device="cuda")
    g = gpu_requantize(fp4, upload_oracle_qtensor(fp4, q), tensor_amax=ta, **kw)
    o = oracle.requantize(q, amax=amax, **kw)
    assert_quant_equal(g, o, what="given amax")


def test_requantize_full_size_dgrad_weight_sampled(fp4):
    # the double-block Dgrad weight of the down projection: W^ [4096, 14336]
    # quantized along its rows in the forward pass, re-quantized along the
    # columns with SR for the Dgrad GEMM; sampled output lines vs the oracle
    from fp4_block_scaled_h16_b200 import workloads
    from parity import sample_lines
    d = workloads.nvfp4_dgrad_down()
    w = d["Wd"].float().numpy()
    q = oracle.quantize(w, NV, double_block=True)
    kw = dict(fmt=NV, rounding=1, rotation=0, double_block=True, seed=0, tensor_id=2)
    g = gpu_requantize(fp4, upload_oracle_qtensor(fp4, q), **kw)
    idx = sample_lines(w.shape[1], 48, 11)
    o = oracle.requantize(q, lines=idx, **kw)
    assert_quant_equal(g, o, lines=idx, what="full-size W^ sampled")
