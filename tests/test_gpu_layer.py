"""Parity of the full Llama-3.1-8B decoder-layer linears at 8192 tokens: QKV
4096 -> 6144, O 4096 -> 4096, fused gate+up 4096 -> 28672 and down
14336 -> 4096 ("Pre-addestramento di Modelli Linguistici di Grandi Dimensioni
con MXFP4", Metodologia: Fprop, Dgrad and Wgrad of every linear in FP4).

Per linear, at full size:
  * the six operands (X and W for Fprop, dY and W^T for Dgrad, dY^T and X^T
    for Wgrad), H16 on all three GEMMs and stochastic rounding on the Wgrad
    operands, quantized by the CUDA path in NVFP4 and in UFP4 and compared
    bit for bit with the oracle on sampled lines (the oracle takes the tensor
    amax over the whole rotated tensor);
  * the three GEMMs in NVFP4 and in UFP4, including the gate+up Dgrad at
    K = 28672, the down Fprop at K = 14336 and the Wgrads at K = 8192,
    compared with the oracle's float64 GEMM on sampled rows and columns within
    |C - C64| <= 1e-5 * sum_k |a_ik b_jk| (+ half a bf16 ulp for bf16 out).
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_quant_equal, assert_within_gemm_bound, oracle_input, sample_lines, untile_lines
from fp4_block_scaled_h16_b200 import workloads

pytestmark = pytest.mark.gpu
NV, UF = 1, 2
H16 = 1


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def rotated_amax(xo: np.ndarray, axis: int) -> float:
    """The oracle's amax of the H16-rotated tensor along `axis`.  Along axis 0
    the lines are the columns: the oracle is given the transposed copy along
    axis 1, the same lines in the same order (the amax has no counter), which
    keeps its reads contiguous."""
    if axis == 1:
        return oracle.tensor_amax(xo, 1, H16)
    return oracle.tensor_amax(np.ascontiguousarray(xo.T), 1, H16)


def gpu_lines(q: dict, lines: np.ndarray) -> dict:
    K, fmt = q["K"], q["format"]
    idx = torch.from_numpy(lines).to(q["codes"].device)
    return dict(codes=q["codes"][idx].cpu().numpy(),
                scales=untile_lines(q["scales"].cpu().numpy(), lines, K, fmt),
                outer=None, tensor_scale=float(q["tensor_scale"].cpu()[0]))


@pytest.mark.parametrize("index", range(len(workloads.LAYER_LINEARS)),
                         ids=[n for n, _, _, _ in workloads.LAYER_LINEARS])
def test_layer_linear_full_size(fp4, index):
    name = workloads.LAYER_LINEARS[index][0]
    d = workloads.layer_linear(name)
    host = {k: oracle_input(v) for k, v in d.items()}
    dev = {k: v.cuda() for k, v in d.items()}
    amax = {}
    qs = {}
    for role, (t, axis, sr) in enumerate(workloads.LAYER_OPERANDS):
        if (t, axis) not in amax:
            amax[(t, axis)] = rotated_amax(host[t], axis)
        R, C = d[t].shape
        L = R if axis == 1 else C
        lines = sample_lines(L, 24, 100 * index + role)
        for fmt in (NV, UF):
            kw = dict(fmt=fmt, rounding=1 if sr else 0, rotation=H16, axis=axis, seed=0,
                      tensor_id=workloads.layer_tensor_id(index, role))
            q = fp4.quantize(dev[t], **kw)
            torch.cuda.synchronize()
            assert fp4.fp4_last_error() == fp4.FP4_OK
            o = oracle.quantize(host[t], amax=amax[(t, axis)], lines=lines, **kw)
            g = gpu_lines(q, lines)
            # g holds the sampled lines only, in the order of `lines`
            assert_quant_equal(g, o, lines=np.arange(len(lines)),
                               what="%s %s axis %d fmt %d" % (name, t, axis, fmt))
            qs[(fmt, role)] = (q, kw)
    for (fmt, gname, ra, rb, out_bf16) in [(f,) + g for f in (NV, UF) for g in workloads.LAYER_GEMMS]:
        (qa, ka), (qb, kb) = qs[(fmt, ra)], qs[(fmt, rb)]
        C = fp4.gemm(qa, qb, fp4.FP4_OUT_BF16 if out_bf16 else fp4.FP4_OUT_F32)
        torch.cuda.synchronize()
        assert fp4.fp4_last_error() == fp4.FP4_OK
        rows = sample_lines(qa["lines"], 40, 7 * index + ra)
        cols = sample_lines(qb["lines"], 40, 7 * index + rb + 1)
        ta, tb = workloads.LAYER_OPERANDS[ra][0], workloads.LAYER_OPERANDS[rb][0]
        oa = oracle.quantize(host[ta], amax=amax[(ta, ka["axis"])], lines=rows, **ka)
        ob = oracle.quantize(host[tb], amax=amax[(tb, kb["axis"])], lines=cols, **kb)
        C64, bound = oracle.gemm(oa, ob)
        sub = C.float()[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].cpu().numpy()
        assert_within_gemm_bound(sub, C64, bound, out_bf16,
                                 what="%s %s fmt %d %s" % (name, gname, fmt, (qa["lines"], qb["lines"], qa["K"])))
        del C
    del dev, qs
    torch.cuda.empty_cache()
