"""Quantizer parity: the CUDA path (through the C ABI) against the CPU oracle,
bit-exact on codes, scales, outer scales and the tensor scale.

Covers every format x rounding x rotation x axis x input dtype on tensors
spanning several tiles with ragged tails, special values, empty inputs, the
stand-alone amax, a caller-given amax, and the full-size Llama-3.1-8B-shaped
workloads on sampled lines.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (assert_quant_equal, gpu_quantize, oracle_quantize, sample_lines)
from fp4_block_scaled_h16_b200 import workloads

pytestmark = pytest.mark.gpu

MX, NV, UF = 0, 1, 2
FORMATS = [(MX, False), (NV, False), (UF, False), (NV, True)]
ROTS = [0, 1, 2, 3, 4]


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def make_input(R, ld, dtype, seed, outliers=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, ld)).astype(np.float32)
    if outliers:
        x[:, rng.choice(ld, 3, replace=False)] *= 50.0
        x[rng.choice(R, 2, replace=False), :] *= 1e-3
    t = torch.from_numpy(x)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def shape_for(axis, db):
    # several tiles and ragged tails: axis 1 has ragged lines (R), axis 0 has
    # ragged lines (C) that are not a multiple of the 64-column tile or of 4
    if axis == 1:
        return 300, 512, 512          # R, C, ld
    return (384, 202, 208) if not db else (384, 200, 200)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("axis", [1, 0])
@pytest.mark.parametrize("rot", ROTS)
@pytest.mark.parametrize("rounding", [0, 1])
@pytest.mark.parametrize("fmt,db", FORMATS)
def test_quantize_sweep(fp4, fmt, db, rounding, rot, axis, dtype):
    R, C, ld = shape_for(axis, db)
    seed = 1000 * fmt + 100 * rounding + 10 * rot + axis + (7 if db else 0)
    x = make_input(R, ld, dtype, seed)
    kw = dict(fmt=fmt, rounding=rounding, rotation=rot, axis=axis, double_block=db,
              seed=0x5EED + seed, tensor_id=3)
    g = gpu_quantize(fp4, x.cuda(), cols=C, **kw)
    o = oracle_quantize(x, cols=C, **kw)
    assert_quant_equal(g, o, what=str(kw))


def special_values(R, C, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, C)).astype(np.float32)
    x[0, :] = 0.0
    x[1, :] = -0.0
    x[2, :] = 0.0
    x[2, 5] = 3.0                          # single nonzero
    x[3, :] = 2.0 ** rng.integers(-10, 10, C)   # exact powers of two
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 0.5, 1.5, 6.5], np.float32)
    x[4, :] = np.resize(ties, C) * np.resize([1, -1], C)
    x[4, ::32] = 4.0                       # MX block scale 1 exactly: the ties stay ties
    x[5, :] = 1e-40                        # subnormal block
    x[6, :] = rng.standard_normal(C) * 1e-38
    x[7, :] = rng.standard_normal(C) * 1e37
    x[8, :] = np.float32(2.0 ** -149)
    x[9, :] = -1e-30
    x[9, 0] = 1.0                          # small negatives rounding to zero keep their sign
    x[10, :] = -0.0
    x[10, ::5] = rng.standard_normal(len(x[10, ::5]))   # -0 inside blocks with a nonzero maximum
    return torch.from_numpy(x)


@pytest.mark.parametrize("rounding", [0, 1])
@pytest.mark.parametrize("fmt,db", FORMATS)
@pytest.mark.parametrize("axis", [1, 0])
def test_special_values(fp4, fmt, db, rounding, axis):
    x = special_values(128, 256, 5 + fmt)
    if axis == 0:
        x = x.t().contiguous()                 # the special rows become special columns
    kw = dict(fmt=fmt, rounding=rounding, rotation=0, axis=axis, double_block=db, seed=9)
    g = gpu_quantize(fp4, x.cuda(), **kw)
    o = oracle_quantize(x, **kw)
    assert_quant_equal(g, o, what="special " + str(kw))


@pytest.mark.parametrize("rot", [0, 1, 4])
def test_special_values_rotated_nv(fp4, rot):
    x = special_values(64, 256, 11)
    kw = dict(fmt=NV, rounding=0, rotation=rot, axis=1, seed=2)
    assert_quant_equal(gpu_quantize(fp4, x.cuda(), **kw), oracle_quantize(x, **kw), what=str(kw))


@pytest.mark.parametrize("shape", [(0, 64), (64, 0), (0, 0)])
@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("axis", [1, 0])
def test_empty_inputs(fp4, shape, fmt, axis):
    x = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    q = fp4.quantize(x, fmt=fmt, axis=axis)
    torch.cuda.synchronize()
    if fmt == NV:
        assert float(q["tensor_scale"].cpu()[0]) == 1.0


@pytest.mark.parametrize("rot", ROTS)
@pytest.mark.parametrize("axis", [1, 0])
def test_amax_matches_oracle(fp4, rot, axis):
    x = make_input(256, 384, "bf16", 40 + rot)
    out = torch.empty(1, dtype=torch.float32, device="cuda")
    xd = x.cuda()
    fp4.fp4_amax(xd, fp4.FP4_IN_BF16, 256, 384, 384, rot, axis, 77, out)
    want = oracle.tensor_amax(np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16)), axis, rot, 77)
    assert np.float32(out.cpu()[0]) == np.float32(want)


def test_caller_given_amax(fp4):
    x = make_input(128, 256, "bf16", 3)
    amax = 2.5 * float(x.float().abs().max())
    t = torch.tensor([amax], dtype=torch.float32, device="cuda")
    kw = dict(fmt=NV, rounding=1, rotation=1, axis=1, seed=4)
    g = gpu_quantize(fp4, x.cuda(), tensor_amax=t, **kw)
    o = oracle_quantize(x, amax=np.float32(amax), **kw)
    assert_quant_equal(g, o, what="given amax")


def check_sampled(fp4, x_cpu, n_lines, sample_seed, **kw):
    """Full-size GPU quantization, compared on sampled lines (the tensor amax
    is taken by the oracle over the whole tensor)."""
    axis = kw["axis"]
    L = x_cpu.shape[0] if axis == 1 else x_cpu.shape[1]
    g = gpu_quantize(fp4, x_cpu.cuda(), **kw)
    lines = sample_lines(L, n_lines, sample_seed)
    o = oracle_quantize(x_cpu, lines=lines, **kw)
    assert_quant_equal(g, o, lines=lines, what="full-size " + str(kw))
    return g


def test_full_tiny_mxfp4(fp4):
    d = workloads.tiny_mxfp4()
    for name, axis in (("A", 1), ("B", 0)):
        kw = dict(fmt=MX, rounding=0, rotation=0, axis=axis)
        g = gpu_quantize(fp4, d[name].cuda(), **kw)
        assert_quant_equal(g, oracle_quantize(d[name], **kw), what=name)


def test_full_nvfp4_fprop_qkv(fp4):
    d = workloads.nvfp4_fprop_qkv()
    for i, name in enumerate(("X", "W")):
        check_sampled(fp4, d[name], 96, i, fmt=NV, rounding=0, rotation=1, axis=1)


def test_full_mxfp4_wgrad_down(fp4):
    d = workloads.mxfp4_wgrad_down()
    for i, name in enumerate(("dY", "H")):
        check_sampled(fp4, d[name], 64, i, fmt=MX, rounding=1, rotation=4, axis=0, seed=0, tensor_id=1 + i)


def test_full_nvfp4_dgrad_double_block(fp4):
    d = workloads.nvfp4_dgrad_down()
    check_sampled(fp4, d["dY"], 96, 0, fmt=NV, rounding=1, rotation=0, axis=1, double_block=True,
                  seed=0, tensor_id=1)
    check_sampled(fp4, d["Wd"], 64, 1, fmt=NV, rounding=1, rotation=0, axis=0, double_block=True,
                  seed=0, tensor_id=2)


@pytest.mark.parametrize("name", ["qkv", "down"])
@pytest.mark.parametrize("fmt", [NV, UF])
def test_layer_linear_operands(fp4, name, fmt):
    """The six operands of one linear (Fprop, Dgrad, Wgrad), H16 on all three
    GEMMs, SR on the Wgrad operands, at 1/4 scale of the layer's shapes."""
    d = workloads.layer_linear(name, scale_dims=4)
    ops = [("X", 1, 0), ("W", 1, 0), ("dY", 1, 0), ("W", 0, 0), ("dY", 0, 1), ("X", 0, 1)]
    for role, (t, axis, sr) in enumerate(ops):
        kw = dict(fmt=fmt, rounding=sr, rotation=1, axis=axis, seed=0, tensor_id=16 + role)
        g = gpu_quantize(fp4, d[t].cuda(), **kw)
        assert_quant_equal(g, oracle_quantize(d[t], **kw), what="%s %s %s" % (name, t, kw))


# The internal amax on the row axis runs as one cooperative launch (amax pass,
# grid barrier, quantize pass); it must give exactly what the two-launch path
# gives: fp4_amax, then fp4_quantize with that amax.  The shapes cover fewer
# stages than CTAs, many lines per stage, a ragged last stage and lines split
# into segments (a line longer than one stage).
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (257, 4096), (1000, 272), (9, 24576)])
@pytest.mark.parametrize("fmt,rounding,rot", [(NV, 0, 1), (NV, 1, 4), (UF, 0, 0), (UF, 1, 3)])
def test_one_launch_amax_matches_two_launches(fp4, shape, fmt, rounding, rot):
    R, C = shape
    if C % (32 if rot in (2, 4) else 16):
        pytest.skip("rotation size does not divide the line")
    x = make_input(R, C, "bf16", seed=R + C, outliers=R >= 2).cuda()
    kw = dict(fmt=fmt, rounding=rounding, rotation=rot, axis=1, seed=11, tensor_id=3)
    one, two = (fp4.alloc_qtensor(R, C, fmt, device=x.device) for _ in range(2))
    for q in (one, two):
        q["scales"].zero_()           # the tiled layout's padding is never written
    fp4.quantize(x, out=one, **kw)
    amax = torch.zeros(1, dtype=torch.float32, device=x.device)
    fp4.fp4_amax(x, fp4.FP4_IN_BF16, R, C, C, rot, 1, 11, amax)
    fp4.quantize(x, tensor_amax=amax, out=two, **kw)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    for key in ("codes", "scales", "tensor_scale"):
        assert torch.equal(one[key].view(torch.uint8), two[key].view(torch.uint8)), key


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("fmt,rounding,rot", [(NV, 0, 1), (UF, 1, 2), (NV, 1, 0)])
def test_one_launch_strided_input_matches_oracle(fp4, dtype, fmt, rounding, rot):
    # the one-launch (internal amax) row path on a view whose row pitch is
    # wider than its rows, in both input types, against the oracle
    R, C, ld = 300, 384, 448
    full = make_input(R, ld, dtype, seed=R + ld + fmt)
    x = full[:, :C]
    kw = dict(fmt=fmt, rounding=rounding, rotation=rot, axis=1, seed=4, tensor_id=6)
    g = gpu_quantize(fp4, full.cuda()[:, :C], cols=C, **kw)
    o = oracle_quantize(x.contiguous(), **kw)
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert_quant_equal(g, o, what="strided one-launch " + str(kw))


# Row lines whose length is an odd multiple of 16 run the row kernel with one
# 16-element unit per thread (the tensor-scaled formats without a 32-rotation);
# the shapes give many lines per stage with a ragged last stage, and lines
# longer than one stage (split into segments, the last one ragged).
@pytest.mark.parametrize("shape", [(300, 272, 280), (7, 48, 48), (5, 4112, 4112)])
@pytest.mark.parametrize("fmt,rounding,rot", [(NV, 0, 0), (NV, 0, 1), (NV, 1, 3), (UF, 0, 1), (UF, 1, 0)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_row_lines_of_odd_sixteens(fp4, shape, fmt, rounding, rot, dtype):
    R, C, ld = shape
    x = make_input(R, ld, dtype, seed=R + C + 10 * fmt + rot, outliers=R >= 2)
    kw = dict(fmt=fmt, rounding=rounding, rotation=rot, axis=1, seed=21, tensor_id=5)
    g = gpu_quantize(fp4, x.cuda(), cols=C, **kw)
    o = oracle_quantize(x, cols=C, **kw)
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert_quant_equal(g, o, what="odd-16 lines %s %s" % (shape, kw))
