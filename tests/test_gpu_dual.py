"""Both-axes quantization (fp4_quantize_both_axes): one launch gives the row
and the column quantizations of a bf16 tensor.  Each output is compared
bit-exactly with the oracle's single-axis quantization (its own rotated amax
and tensor scale) on tensors spanning several tiles with a ragged last row
tile and a row pitch wider than the row, on special values, and at the
Llama-3.1-8B layer sizes on sampled lines, with the single-axis calls beside
it bit for bit."""
import numpy as np
import pytest
import torch

from parity import assert_quant_equal, oracle_quantize, sample_lines, untile
from fp4_block_scaled_h16_b200 import workloads

pytestmark = pytest.mark.gpu

NV, UF = 1, 2


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def host(q):
    L, K, fmt = q["lines"], q["K"], q["format"]
    return dict(codes=q["codes"].cpu().numpy(), scales=untile(q["scales"].cpu().numpy(), L, K, fmt),
                outer=None, tensor_scale=float(q["tensor_scale"].cpu()[0]))


def both(fp4, x_dev, cols=None, **kw):
    if cols is not None and cols != x_dev.shape[1]:
        x_dev = x_dev[:, :cols]
    qr, qc = fp4.quantize_both_axes(x_dev, **kw)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    return qr, qc


def make_input(R, ld, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, ld)).astype(np.float32)
    x[:, rng.choice(ld, 3, replace=False)] *= 50.0
    x[rng.choice(R, 2, replace=False), :] *= 1e-3
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("rr,rc", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("rot", [0, 1])
@pytest.mark.parametrize("fmt", [NV, UF])
def test_both_axes_sweep(fp4, fmt, rot, rr, rc):
    # 400 rows: three whole row tiles and a ragged fourth; 320 columns: five
    # column tiles; row pitch 336
    R, C, ld = 400, 320, 336
    seed = 100 * fmt + 10 * rot + 2 * rr + rc
    x = make_input(R, ld, seed)
    kw = dict(fmt=fmt, rotation=rot, seed=0x5EED + seed, rounding_rows=rr, tensor_id_rows=5,
              rounding_cols=rc, tensor_id_cols=6)
    qr, qc = both(fp4, x.cuda()[:, :C], **kw)
    xs = x[:, :C].contiguous()
    orow = oracle_quantize(xs, fmt, rounding=rr, rotation=rot, axis=1, seed=0x5EED + seed, tensor_id=5)
    ocol = oracle_quantize(xs, fmt, rounding=rc, rotation=rot, axis=0, seed=0x5EED + seed, tensor_id=6)
    assert_quant_equal(host(qr), orow, what="rows " + str(kw))
    assert_quant_equal(host(qc), ocol, what="columns " + str(kw))


@pytest.mark.parametrize("rounding", [0, 1])
def test_both_axes_special_values(fp4, rounding):
    from test_gpu_quant import special_values
    x = special_values(128, 256, 23).to(torch.bfloat16)
    # the special rows along the rows, and the same values as columns of the transpose
    for t in (x, x.t().contiguous()):
        kw = dict(fmt=NV, rotation=0, seed=9, rounding_rows=rounding, tensor_id_rows=1,
                  rounding_cols=rounding, tensor_id_cols=2)
        qr, qc = both(fp4, t.cuda(), **kw)
        assert_quant_equal(host(qr), oracle_quantize(t, NV, rounding=rounding, axis=1, seed=9, tensor_id=1),
                           what="special rows")
        assert_quant_equal(host(qc), oracle_quantize(t, NV, rounding=rounding, axis=0, seed=9, tensor_id=2),
                           what="special columns")


def test_both_axes_all_zero_tensor(fp4):
    x = torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda")
    qr, qc = both(fp4, x, fmt=NV, rotation=1)
    for q in (qr, qc):
        assert float(q["tensor_scale"].cpu()[0]) == 1.0
        assert int(q["codes"].abs().sum()) == 0


def test_both_axes_empty(fp4):
    for shape in ((0, 64), (32, 0)):
        x = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        qr, qc = both(fp4, x, fmt=NV)
        assert float(qr["tensor_scale"].cpu()[0]) == 1.0 and float(qc["tensor_scale"].cpu()[0]) == 1.0


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=torch.float32), 8), (dict(fmt=0), 8), (dict(rotation=2), 8), (dict(rotation=3), 8),
    (dict(cols=96), 2), (dict(rows=24), 2),
])
def test_both_axes_rejects(fp4, kw, status):
    R, C = kw.get("rows", 64), kw.get("cols", 128)
    x = torch.zeros((R, C), dtype=kw.get("dtype", torch.bfloat16), device="cuda")
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.quantize_both_axes(x, fmt=kw.get("fmt", NV), rotation=kw.get("rotation", 1))
    assert e.value.status == status


@pytest.mark.parametrize("name", ["qkv", "gate_up"])
def test_both_axes_layer_sizes(fp4, name):
    """X, W and dY of one Llama-3.1-8B linear at T = 8192 with the layer step's
    roundings and stochastic-rounding streams: the both-axes outputs equal the
    two single-axis calls bit for bit on every line, and the oracle on
    sampled lines."""
    index = [n for n, _, _, _ in workloads.LAYER_LINEARS].index(name)
    d = workloads.layer_linear(name)
    roles = {(tn, axis): (role, sr) for role, (tn, axis, sr) in enumerate(workloads.LAYER_OPERANDS)}
    for k, tn in enumerate(("X", "W", "dY")):
        x = d[tn].cuda()
        rrole, rsr = roles[(tn, 1)]
        crole, csr = roles[(tn, 0)]
        kw = dict(fmt=NV, rotation=1, seed=0, rounding_rows=int(rsr),
                  tensor_id_rows=workloads.layer_tensor_id(index, rrole),
                  rounding_cols=int(csr), tensor_id_cols=workloads.layer_tensor_id(index, crole))
        qr, qc = both(fp4, x, **kw)
        sr = fp4.quantize(x, NV, kw["rounding_rows"], 1, axis=1, seed=0, tensor_id=kw["tensor_id_rows"])
        sc = fp4.quantize(x, NV, kw["rounding_cols"], 1, axis=0, seed=0, tensor_id=kw["tensor_id_cols"])
        torch.cuda.synchronize()
        for a, b in ((qr, sr), (qc, sc)):
            assert torch.equal(a["codes"], b["codes"]), (name, tn)
            assert torch.equal(a["scales"], b["scales"]), (name, tn)
            assert torch.equal(a["tensor_scale"], b["tensor_scale"]), (name, tn)
        del sr, sc
        R, C = d[tn].shape
        hr, hc = host(qr), host(qc)
        lr, lc = sample_lines(R, 24, k), sample_lines(C, 24, 10 + k)
        assert_quant_equal(hr, oracle_quantize(d[tn], NV, rounding=kw["rounding_rows"], rotation=1, axis=1, seed=0,
                                               tensor_id=kw["tensor_id_rows"], lines=lr), lines=lr,
                           what="%s.%s rows" % (name, tn))
        assert_quant_equal(hc, oracle_quantize(d[tn], NV, rounding=kw["rounding_cols"], rotation=1, axis=0, seed=0,
                                               tensor_id=kw["tensor_id_cols"], lines=lc), lines=lc,
                           what="%s.%s columns" % (name, tn))


@pytest.mark.parametrize("shape", [(16, 64), (144, 128), (48, 192), (272, 64)])
@pytest.mark.parametrize("rr,rc", [(0, 1), (1, 0)])
def test_both_axes_small_and_ragged(fp4, shape, rr, rc):
    # fewer rows than one 128-row tile, a ragged second tile, one column tile
    R, C = shape
    x = make_input(R, C, 7 * R + C + rr)
    kw = dict(fmt=NV, rotation=1, seed=11, rounding_rows=rr, tensor_id_rows=3, rounding_cols=rc, tensor_id_cols=4)
    qr, qc = both(fp4, x.cuda(), **kw)
    assert_quant_equal(host(qr), oracle_quantize(x, NV, rounding=rr, rotation=1, axis=1, seed=11, tensor_id=3),
                       what="rows %s" % (shape,))
    assert_quant_equal(host(qc), oracle_quantize(x, NV, rounding=rc, rotation=1, axis=0, seed=11, tensor_id=4),
                       what="columns %s" % (shape,))
