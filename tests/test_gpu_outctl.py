"""OutControl ("TetraJet-v2" 2.C) on the GPU against the oracle: the
calibration statistic (per-channel amax), the split of an operand into its
NVFP4 part (channels zeroed) and its E4M3 part (channels gathered), bit for
bit, and the split GEMM within |C - C64| <= 1e-5 sum |a b| (+ half a bf16 ulp
for bf16 output), on oracle operands and through the whole path on the
QKV-shaped Fprop with its outlier channels.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_quant_equal, assert_within_gemm_bound, oracle_input, sample_lines, tile, untile

pytestmark = pytest.mark.gpu
NV = 1


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def make(R, C, seed, dtype=torch.bfloat16, outliers=6):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, C)).astype(np.float32)
    x[:, rng.choice(C, outliers, replace=False)] *= 64.0
    return torch.from_numpy(x).to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", [(300, 512), (7, 4096), (1000, 272)])
def test_channel_amax(fp4, dtype, shape):
    x = make(*shape, seed=shape[0], dtype=dtype)
    got = fp4.channel_amax(x.cuda()).cpu().numpy()
    want = np.abs(oracle.widen(oracle_input(x))).max(axis=0)
    assert (got.view(np.uint32) == want.view(np.uint32)).all()


def gpu_split(fp4, q):
    torch.cuda.synchronize()
    q4, q8 = q["fp4"], q["fp8"]
    L, K = q4["lines"], q4["K"]
    return dict(codes=q4["codes"].cpu().numpy(), scales=untile(q4["scales"].cpu().numpy(), L, K, NV), outer=None,
                tensor_scale=float(q4["tensor_scale"].cpu()[0])), q8["codes"].cpu().numpy(), float(q8["scale"].cpu()[0])


@pytest.mark.parametrize("n", [0, 37, 128, 200])
@pytest.mark.parametrize("rounding,rotation", [(0, 0), (1, 1), (0, 3)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_split_matches_oracle(fp4, n, rounding, rotation, dtype):
    R, C = 300, 512
    x = make(R, C, seed=n + rotation, dtype=dtype)
    rng = np.random.default_rng(n)
    ch = np.sort(rng.choice(C, n, replace=False)).astype(np.int32)
    k8 = (n + 127) // 128 * 128
    q = fp4.outctl_quantize(x.cuda(), torch.from_numpy(ch).cuda(), k8, rounding=rounding, rotation=rotation,
                            seed=3, tensor_id=5)
    g4, g8, gs8 = gpu_split(fp4, q)
    assert fp4.fp4_last_error() == fp4.FP4_OK
    o = oracle.outctl_quantize(oracle_input(x), ch, k8, rounding=rounding, rotation=rotation, seed=3, tensor_id=5)
    assert_quant_equal(g4, o["fp4"], what="fp4 part")
    assert np.float32(gs8) == np.float32(o["fp8"]["scale"])
    assert (g8[:, :k8] == o["fp8"]["codes"]).all()


def upload(fp4, o):
    q4 = o["fp4"]
    L, K = q4["codes"].shape[0], q4["K"]
    t4 = dict(codes=torch.from_numpy(np.ascontiguousarray(q4["codes"])).cuda(),
              scales=torch.from_numpy(tile(q4["scales"], NV, fp4.fp4_scales_bytes(L, K, NV))).cuda(),
              outer=None, tensor_scale=torch.tensor([q4["tensor_scale"]], dtype=torch.float32).cuda(),
              lines=L, K=K, format=NV, double_block=False)
    q8 = o["fp8"]
    t8 = dict(codes=torch.from_numpy(np.ascontiguousarray(q8["codes"])).cuda(),
              scale=torch.tensor([q8["scale"]], dtype=torch.float32).cuda(), K=q8["K"])
    return dict(fp4=t4, fp8=t8)


@pytest.mark.parametrize("out_bf16", [False, True])
@pytest.mark.parametrize("shape", [(128, 128, 256, 128), (256, 384, 512, 256), (128, 256, 384, 128),
                                   (384, 128, 1024, 0), (1280, 1280, 2048, 384)])
def test_split_gemm_on_oracle_operands(fp4, shape, out_bf16):
    M, N, K, K8 = shape
    a, b = make(M, K, M + K, torch.float32), make(N, K, N + 2 * K, torch.float32) * 0.05
    ch = oracle.outctl_channels(oracle_input(a), min(K8, 100) / K) if K8 else np.zeros(0, np.int32)
    oa = oracle.outctl_quantize(oracle_input(a), ch, K8)
    ob = oracle.outctl_quantize(oracle_input(b), ch, K8, rounding=1, seed=2, tensor_id=1)
    C64, bound = oracle.gemm_outctl(oa, ob)
    C = fp4.gemm_outctl(upload(fp4, oa), upload(fp4, ob), fp4.FP4_OUT_BF16 if out_bf16 else fp4.FP4_OUT_F32)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    assert_within_gemm_bound(C.float().cpu().numpy(), C64, bound, out_bf16, what=str(shape))


def test_fprop_qkv_with_outcontrol(fp4):
    """The QKV Fprop (X 8192 x 4096 with its outlier channels, W 6144 x 4096):
    calibration on X, the top 10% channels in FP8; sampled rows and columns of
    C against the oracle, and the split closer to the exact product than plain
    NVFP4 on them."""
    from fp4_block_scaled_h16_b200 import workloads
    d = workloads.nvfp4_fprop_qkv()
    X, W = d["X"].cuda(), d["W"].cuda()
    ch = fp4.outctl_channels(fp4.channel_amax(X), 0.10)
    ch_host = oracle.outctl_channels(oracle_input(d["X"]), 0.10)
    assert (ch.cpu().numpy() == ch_host).all()
    qx, qw = fp4.outctl_quantize(X, ch), fp4.outctl_quantize(W, ch)
    C = fp4.gemm_outctl(qx, qw, fp4.FP4_OUT_BF16)
    torch.cuda.synchronize()
    assert fp4.fp4_last_error() == fp4.FP4_OK
    rows, cols = sample_lines(8192, 48, 1), sample_lines(6144, 48, 2)
    k8 = qx["fp8"]["K"]
    ox = oracle.outctl_quantize(oracle_input(d["X"]), ch_host, k8, lines=rows)
    ow = oracle.outctl_quantize(oracle_input(d["W"]), ch_host, k8, lines=cols)
    C64, bound = oracle.gemm_outctl(ox, ow)
    sub = C.float()[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].cpu().numpy()
    assert_within_gemm_bound(sub, C64, bound, True, what="fprop qkv outcontrol")
    exact = d["X"].double().numpy()[rows] @ d["W"].double().numpy()[cols].T
    plain = fp4.gemm(fp4.quantize(X, NV), fp4.quantize(W, NV), fp4.FP4_OUT_F32)
    plain_sub = plain[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].double().cpu().numpy()
    assert np.linalg.norm(sub - exact) < np.linalg.norm(plain_sub - exact)


def test_bad_channel_index_is_reported(fp4):
    x = make(128, 256, 1).cuda()
    ch = torch.tensor([3, 77, 300], dtype=torch.int32, device="cuda")       # 300 is past the columns
    fp4.outctl_quantize(x, ch, 128)
    assert fp4.fp4_last_error() == fp4.FP4_ERR_INVALID_ARG
    fp4.outctl_quantize(x, ch[:2], 128)
    assert fp4.fp4_last_error() == fp4.FP4_OK
