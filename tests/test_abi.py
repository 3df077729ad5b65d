"""The C ABI library loads, exports every entry point include/fp4.h declares,
and validates arguments on the host (no GPU needed, nothing launched)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp4.h")

fp4 = pytest.importorskip("fp4_block_scaled_h16_b200.fp4", reason="libfp4.so not built")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 8
    lib = ctypes.CDLL(fp4.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(fp4.EXPORTS)


def test_status_strings():
    assert fp4.fp4_status_string(0) == "FP4_OK"
    assert fp4.fp4_status_string(7) == "FP4_ERR_TIMEOUT"
    assert fp4.fp4_status_string(99) == "FP4_ERR_UNKNOWN"


def test_scales_bytes_and_workspace():
    assert fp4.fp4_scales_bytes(0, 64, fp4.FP4_NVFP4) == 0
    assert fp4.fp4_scales_bytes(1, 16, fp4.FP4_NVFP4) == 128 * 4
    assert fp4.fp4_scales_bytes(129, 4096, fp4.FP4_NVFP4) == 256 * 256
    assert fp4.fp4_scales_bytes(256, 512, fp4.FP4_MXFP4) == 256 * 16
    assert fp4.fp4_quantize_workspace_size(fp4.FP4_NVFP4, False, False) == 256
    assert fp4.fp4_quantize_workspace_size(fp4.FP4_NVFP4, False, True) == 0
    assert fp4.fp4_quantize_workspace_size(fp4.FP4_NVFP4, True, False) == 0
    assert fp4.fp4_quantize_workspace_size(fp4.FP4_MXFP4, False, False) == 0
    with pytest.raises(fp4.Fp4Error):
        fp4.fp4_quantize_workspace_size(7, False, False)


ADDR = 1 << 20       # a fake, 16-byte aligned address: validation fails before any use


def q(**kw):
    args = dict(x=ADDR, in_dtype=fp4.FP4_IN_BF16, rows=256, cols=512, ld=512, fmt=fp4.FP4_NVFP4,
                rounding=fp4.FP4_RTNE, rotation=fp4.FP4_ROT_H16, axis=1, double_block=0, seed=0,
                tensor_id=0, tensor_amax=None, codes=ADDR, scales=ADDR, outer_scales=None,
                tensor_scale=ADDR, workspace=ADDR, workspace_bytes=256)
    args.update(kw)
    return fp4._lib.fp4_quantize(args["x"], args["in_dtype"], args["rows"], args["cols"], args["ld"],
                                 args["fmt"], args["rounding"], args["rotation"], args["axis"],
                                 args["double_block"], args["seed"], args["tensor_id"], args["tensor_amax"],
                                 args["codes"], args["scales"], args["outer_scales"], args["tensor_scale"],
                                 args["workspace"], args["workspace_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(in_dtype=5), 1), (dict(fmt=3), 1), (dict(rounding=2), 1), (dict(rotation=9), 1),
    (dict(axis=2), 1), (dict(rows=-1), 1), (dict(ld=100), 1), (dict(x=None), 1),
    (dict(codes=None), 1), (dict(tensor_scale=None), 1), (dict(double_block=1, fmt=fp4.FP4_MXFP4), 1),
    (dict(double_block=1, outer_scales=None), 1),
    (dict(x=ADDR + 8), 3), (dict(ld=516, cols=512), 3), (dict(codes=ADDR + 4), 3),
    (dict(cols=500, ld=512), 2), (dict(fmt=fp4.FP4_MXFP4, cols=496, ld=512), 2),
    (dict(rotation=fp4.FP4_ROT_H32, cols=496, ld=512), 2),
    (dict(double_block=1, outer_scales=ADDR, cols=448, ld=448), 2),
    (dict(axis=0, rows=200), 2),
    (dict(workspace=None), 4), (dict(workspace_bytes=16), 4),
])
def test_quantize_host_validation(kw, status):
    assert q(**kw) == status


def g(**kw):
    args = dict(fmt=fp4.FP4_NVFP4, db=0, a=ADDR, sa=ADDR, oa=None, ta=ADDR, b=ADDR, sb=ADDR, ob=None, tb=ADDR,
                M=256, N=256, K=512, c=ADDR, out=fp4.FP4_OUT_BF16, ldc=256, ws=None, wsb=0)
    args.update(kw)
    return fp4._lib.fp4_gemm(args["fmt"], args["db"], args["a"], args["sa"], args["oa"], args["ta"], args["b"],
                             args["sb"], args["ob"], args["tb"], args["M"], args["N"], args["K"], args["c"],
                             args["out"], args["ldc"], args["ws"], args["wsb"], None)


UFP4_WS = 2 * (256 * 2 * 512 + 256 * 4 * 512 // 16)     # both operands' split codes + scales at M = N = 256, K = 512


@pytest.mark.parametrize("kw,status", [
    (dict(fmt=7), 1), (dict(fmt=fp4.FP4_UFP4), 4), (dict(fmt=fp4.FP4_UFP4, ws=ADDR, wsb=1024), 4),
    (dict(fmt=fp4.FP4_UFP4, ws=ADDR + 8, wsb=UFP4_WS), 3), (dict(fmt=fp4.FP4_UFP4, ta=None, ws=ADDR, wsb=UFP4_WS), 1),
    (dict(fmt=fp4.FP4_UFP4, db=1, oa=ADDR, ob=ADDR), 1), (dict(out=3), 1), (dict(ldc=100), 1),
    (dict(M=-128), 1), (dict(a=None), 1), (dict(ta=None), 1), (dict(db=1, fmt=fp4.FP4_MXFP4), 1),
    (dict(M=200), 2), (dict(N=192), 2), (dict(K=320), 2), (dict(K=0), 2),
    (dict(a=ADDR + 8), 3), (dict(ldc=260), 3),
    (dict(db=1, oa=ADDR + 8, ob=ADDR), 3), (dict(db=1, oa=ADDR, ob=ADDR + 4), 3),
    (dict(db=1, oa=None, ob=ADDR), 1),
])
def test_gemm_host_validation(kw, status):
    assert g(**kw) == status


def test_empty_gemm_is_a_no_op():
    assert g(M=0) == 0 and g(N=0, ldc=0) == 0


def rq(**kw):
    args = dict(sc=ADDR, ss=ADDR, so=None, sts=ADDR, lines=256, K=512, sfmt=fp4.FP4_NVFP4, sdb=0,
                fmt=fp4.FP4_NVFP4, rounding=fp4.FP4_SR, rotation=fp4.FP4_ROT_NONE, db=0, seed=0, tid=0,
                amax=None, codes=ADDR, scales=ADDR, outer=None, ts=ADDR, ws=ADDR, wsb=256)
    args.update(kw)
    a = args
    return fp4._lib.fp4_requantize(a["sc"], a["ss"], a["so"], a["sts"], a["lines"], a["K"], a["sfmt"], a["sdb"],
                                   a["fmt"], a["rounding"], a["rotation"], a["db"], a["seed"], a["tid"], a["amax"],
                                   a["codes"], a["scales"], a["outer"], a["ts"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(sfmt=3), 1), (dict(fmt=5), 1), (dict(rounding=2), 1), (dict(rotation=7), 1), (dict(sdb=2), 1),
    (dict(sdb=1, sfmt=fp4.FP4_MXFP4), 1), (dict(db=1, fmt=fp4.FP4_UFP4), 1), (dict(lines=-1), 1),
    (dict(sc=None), 1), (dict(sts=None), 1), (dict(sdb=1, so=None), 1), (dict(codes=None), 1),
    (dict(db=1, outer=None), 1), (dict(ts=None), 1),
    (dict(K=520), 2), (dict(sfmt=fp4.FP4_MXFP4, K=528), 2), (dict(sdb=1, so=ADDR, K=576), 2),
    (dict(lines=264), 2), (dict(fmt=fp4.FP4_MXFP4, lines=272), 2), (dict(rotation=fp4.FP4_ROT_H32, lines=272), 2),
    (dict(db=1, outer=ADDR, lines=320), 2),
    (dict(sc=ADDR + 8), 3), (dict(codes=ADDR + 4), 3), (dict(so=ADDR + 2, sdb=1), 3),
    (dict(ws=None), 4), (dict(wsb=8), 4),
])
def test_requantize_host_validation(kw, status):
    assert rq(**kw) == status


@pytest.mark.skipif(torch.cuda.is_available(), reason="an empty call writes tensor_scale: the fake address "
                    "must never reach a GPU")
def test_empty_requantize_is_a_no_op_without_gpu_work():
    assert rq(lines=0, sc=None, ss=None, codes=None, scales=None, ws=None) == fp4.FP4_ERR_NO_DEVICE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU answer")
def test_valid_call_without_gpu_reports_no_device():
    assert q() == fp4.FP4_ERR_NO_DEVICE
    assert g() == fp4.FP4_ERR_NO_DEVICE


def both(**kw):
    a = dict(x=ADDR, dt=fp4.FP4_IN_BF16, rows=256, cols=512, ld=512, fmt=fp4.FP4_NVFP4, rotation=fp4.FP4_ROT_H16,
             seed=0, rr=fp4.FP4_RTNE, idr=0, cr=ADDR, sr=ADDR, tr=ADDR, rc=fp4.FP4_SR, idc=1, cc=ADDR, sc=ADDR,
             tc=ADDR, ws=ADDR, wsb=256)
    a.update(kw)
    return fp4._lib.fp4_quantize_both_axes(a["x"], a["dt"], a["rows"], a["cols"], a["ld"], a["fmt"], a["rotation"],
                                           a["seed"], a["rr"], a["idr"], a["cr"], a["sr"], a["tr"], a["rc"], a["idc"],
                                           a["cc"], a["sc"], a["tc"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(dt=5), 1), (dict(fmt=3), 1), (dict(rr=2), 1), (dict(rc=-1), 1), (dict(rotation=9), 1),
    (dict(x=None), 1), (dict(cr=None), 1), (dict(sc=None), 1), (dict(tr=None), 1), (dict(tc=None), 1),
    (dict(rows=-1), 1), (dict(ld=500), 1),
    (dict(dt=fp4.FP4_IN_F32), 8), (dict(fmt=fp4.FP4_MXFP4), 8), (dict(rotation=fp4.FP4_ROT_H32), 8),
    (dict(rotation=fp4.FP4_ROT_RH16), 8),
    (dict(cols=480, ld=512), 2), (dict(rows=200), 2),
    (dict(x=ADDR + 8), 3), (dict(cc=ADDR + 4), 3), (dict(tr=ADDR + 2), 3),
    (dict(ws=None), 4), (dict(wsb=16), 4),
    (dict(), fp4.FP4_ERR_NO_DEVICE),
])
def test_quantize_both_axes_host_validation(kw, status):
    assert both(**kw) == status


def rot(**kw):
    a = dict(x=ADDR, dt=fp4.FP4_IN_BF16, rows=64, cols=256, ld=256, rotation=fp4.FP4_ROT_H16, axis=1, seed=0,
             y=ADDR, ldy=256)
    a.update(kw)
    return fp4._lib.fp4_rotate(a["x"], a["dt"], a["rows"], a["cols"], a["ld"], a["rotation"], a["axis"], a["seed"],
                               a["y"], a["ldy"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(dt=3), 1), (dict(rotation=0), 1), (dict(rotation=9), 1), (dict(ldy=128), 1), (dict(y=None), 1),
    (dict(axis=0), 8), (dict(cols=248, ld=256), 2), (dict(rotation=fp4.FP4_ROT_H32, cols=240, ld=256), 2),
    (dict(y=ADDR + 8), 3), (dict(ldy=260), 3), (dict(x=ADDR + 2), 3),
])
def test_rotate_host_validation(kw, status):
    assert rot(**kw) == status


def mn(**kw):
    a = dict(x=ADDR, dt=fp4.FP4_IN_BF16, rows=64, cols=256, ld=256, fmt=fp4.FP4_NVFP4, rounding=0, p=2, c=2.0, seed=0,
             tid=0, codes=ADDR, scales=ADDR, ts=ADDR, rho=ADDR, ws=ADDR, wsb=256)
    a.update(kw)
    return fp4._lib.fp4_mxnorm_quantize(a["x"], a["dt"], a["rows"], a["cols"], a["ld"], a["fmt"], a["rounding"],
                                        a["p"], a["c"], a["seed"], a["tid"], a["codes"], a["scales"], a["ts"],
                                        a["rho"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(dt=4), 1), (dict(fmt=5), 1), (dict(rounding=3), 1), (dict(p=0), 1), (dict(p=3), 1), (dict(c=0.0), 1),
    (dict(c=-1.0), 1), (dict(c=float("nan")), 1), (dict(c=float("inf")), 1), (dict(ts=None), 1), (dict(rho=None), 1),
    (dict(codes=None), 1), (dict(ld=128), 1),
    (dict(cols=248, ld=256), 2), (dict(fmt=fp4.FP4_MXFP4, cols=240, ld=256), 2), (dict(cols=16400, ld=16400), 2),
    (dict(cols=0), 2),
    (dict(x=ADDR + 4), 3), (dict(codes=ADDR + 8), 3), (dict(rho=ADDR + 2), 3), (dict(ws=ADDR + 4), 3),
    (dict(ws=None), 4), (dict(wsb=64), 4),
])
def test_mxnorm_host_validation(kw, status):
    assert mn(**kw) == status


def test_gemm_workspace_size():
    assert fp4.fp4_gemm_workspace_size(fp4.FP4_NVFP4, False, 256, 256, 512) == 0
    assert fp4.fp4_gemm_workspace_size(fp4.FP4_MXFP4, False, 256, 256, 512) == 0
    assert fp4.fp4_gemm_workspace_size(fp4.FP4_UFP4, False, 256, 256, 512) == UFP4_WS
    # K is rounded up to 256 per split part
    assert fp4.fp4_gemm_workspace_size(fp4.FP4_UFP4, False, 128, 128, 384) == 2 * (128 * 2 * 512 + 128 * 4 * 512 // 16)
    with pytest.raises(fp4.Fp4Error):
        fp4.fp4_gemm_workspace_size(9, False, 1, 1, 1)


def oq(**kw):
    a = dict(x=ADDR, dt=fp4.FP4_IN_BF16, rows=64, cols=256, ld=256, ch=ADDR, n=20, k8=128, rounding=0, rotation=0,
             seed=0, tid=0, codes=ADDR, scales=ADDR, ts=ADDR, codes8=ADDR, s8=ADDR, ws=ADDR, wsb=4096)
    a.update(kw)
    return fp4._lib.fp4_outctl_quantize(a["x"], a["dt"], a["rows"], a["cols"], a["ld"], a["ch"], a["n"], a["k8"],
                                        a["rounding"], a["rotation"], a["seed"], a["tid"], a["codes"], a["scales"],
                                        a["ts"], a["codes8"], a["s8"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(dt=2), 1), (dict(rounding=5), 1), (dict(n=-1), 1), (dict(n=200, k8=128), 1), (dict(ch=None), 1),
    (dict(ts=None), 1), (dict(s8=None), 1), (dict(codes8=None), 1), (dict(codes=None), 1),
    (dict(cols=248, ld=256), 2), (dict(k8=100), 2), (dict(rotation=2, cols=240, ld=256), 2),
    (dict(codes8=ADDR + 8), 3), (dict(ch=ADDR + 2), 3), (dict(ws=ADDR + 4), 3),
    (dict(ws=None), 4), (dict(wsb=100), 4),
])
def test_outctl_quantize_host_validation(kw, status):
    assert oq(**kw) == status


def og(**kw):
    a = dict(a=ADDR, sa=ADDR, ta=ADDR, b=ADDR, sb=ADDR, tb=ADDR, a8=ADDR, s8a=ADDR, b8=ADDR, s8b=ADDR, M=256, N=256,
             K=512, K8=128, c=ADDR, out=fp4.FP4_OUT_BF16, ldc=256)
    a.update(kw)
    return fp4._lib.fp4_gemm_outctl(a["a"], a["sa"], a["ta"], a["b"], a["sb"], a["tb"], a["a8"], a["s8a"], a["b8"],
                                    a["s8b"], a["M"], a["N"], a["K"], a["K8"], a["c"], a["out"], a["ldc"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(out=2), 1), (dict(K8=-128), 1), (dict(ldc=100), 1), (dict(a8=None), 1), (dict(s8b=None), 1),
    (dict(ta=None), 1), (dict(M=200), 2), (dict(K8=100), 2), (dict(K=0), 2), (dict(a8=ADDR + 8), 3),
    (dict(c=ADDR + 4), 3),
])
def test_gemm_outctl_host_validation(kw, status):
    assert og(**kw) == status


def test_outctl_workspace_size():
    assert fp4.fp4_outctl_workspace_size(4096) == 272 + 4096 // 8
    assert fp4.fp4_outctl_workspace_size(0) == 272
