"""CPU oracle for block-scaled FP4 quantization and the block-scaled FP4 GEMM.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the library package
(``fp4_block_scaled_h16_b200``) never does, and this package never imports it.

The quantizer is plain C (``fp4_oracle.c``, compiled with FMA contraction off),
called through ctypes; the GEMM is the plain definition: dequantize both
operands exactly into float64 and take their float64 matrix product, with the
per-element bound sum_k |a_ik * b_jk| beside it.

Sources (page titles, sections):
  * E2M1 grid, RTNE, shrinkage: "Ripensare il Bias di Shrinkage nel Pretraining
    di LLM in FP4", Problematica, Metodologia 1; UFP4: Metodologia 2.
  * MXFP4, H16/H32, random Hadamard: "Pre-addestramento di Modelli Linguistici
    di Grandi Dimensioni con MXFP4", Metodologia.
  * NVFP4 16-groups, double block 128/16, SR, 1x16 transposed groups:
    "TetraJet-v2", section 2.A.
  * Fprop / Dgrad / Wgrad GEMMs on FP4 operands: the MXFP4 page, Metodologia.

Parity unpinned (readings the pages do not fix, pinned only between this
oracle and the CUDA path): the binary32 operation order of the NVFP4 / UFP4 /
double-block scale, the H32 normalisation constant, the Philox counter layout
for SR and the random signs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

MXFP4, NVFP4, UFP4 = 0, 1, 2
RTNE, SR = 0, 1
ROT_NONE, ROT_H16, ROT_H32, ROT_RH16, ROT_RH32 = 0, 1, 2, 3, 4
IN_F32, IN_BF16 = 0, 1

E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def build(force: bool = False) -> str:
    """Compile fp4_oracle.c into liboracle.so next to it (gcc, no FMA contraction)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
                           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, u64, u32, f32, i32 = (ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32,
                                   ctypes.c_float, ctypes.c_int)
        L.orc_philox4x32_10.argtypes = [P, P, P]
        L.orc_rht_signs.argtypes = [u64, i32, P]
        L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_ufp4_value.argtypes = [ctypes.c_uint8]
        L.orc_ufp4_value.restype = ctypes.c_double
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_e4m3_encode.argtypes = [f32]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e2m1_rtne_index.argtypes = [f32]
        L.orc_ufp4_rtne_index.argtypes = [f32]
        L.orc_rotate_block.argtypes = [P, i32, P]
        L.orc_c32.restype = f32
        L.orc_tensor_amax.argtypes = [P, i32, i64, i64, i64, i32, i32, u64, i64, i64]
        L.orc_tensor_amax.restype = f32
        L.orc_tensor_scale.argtypes = [f32, i32]
        L.orc_tensor_scale.restype = f32
        L.orc_quantize_lines.argtypes = [P, i32, i64, i64, i64, i32, i32, i32, i32, i32,
                                         u64, u32, f32, i64, i64, P, P, P]
        L.orc_dequantize.argtypes = [P, P, P, f32, i64, i64, i32, i32, P]
        L.orc_pairwise_sum.argtypes = [P, i64]
        L.orc_pairwise_sum.restype = ctypes.c_double
        L.orc_mxnorm_rho.argtypes = [P, i32, i64, i64, i64, i32, i32, ctypes.c_double, i64, i64, P, P]
        L.orc_fp8_encode_array.argtypes = [P, i64, f32, P]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, min(os.cpu_count() or 1, 32))


# --------------------------------------------------------------------------- scalars

def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def rht_signs(seed: int, n: int) -> np.ndarray:
    d = np.zeros(n, dtype=np.float32)
    lib().orc_rht_signs(seed, n, _ptr(d))
    return d


def rotate_block(x, signs=None) -> np.ndarray:
    b = np.array(x, dtype=np.float32)
    d = None if signs is None else np.ascontiguousarray(signs, dtype=np.float32)
    lib().orc_rotate_block(_ptr(b), len(b), None if d is None else _ptr(d))
    return b


def c32() -> float:
    return lib().orc_c32()


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(code)


def e4m3_encode(s: float) -> int:
    return lib().orc_e4m3_encode(s)


def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(code)


def ufp4_value(code: int) -> float:
    return lib().orc_ufp4_value(code)


def e2m1_rtne_index(u: float) -> int:
    return lib().orc_e2m1_rtne_index(u)


def ufp4_rtne_index(u: float) -> int:
    return lib().orc_ufp4_rtne_index(u)


def tensor_scale(amax: float, fmt: int) -> float:
    return lib().orc_tensor_scale(amax, fmt)


# --------------------------------------------------------------------------- tensors

def _as_input(x: np.ndarray):
    if x.dtype == np.float32:
        return IN_F32
    if x.dtype == np.uint16:           # bfloat16 bit patterns
        return IN_BF16
    raise TypeError("oracle input must be float32 or uint16 (bf16 bits), got %s" % x.dtype)


def _chunks(l0: int, l1: int, threads: int):
    n = l1 - l0
    if n <= 0:
        return []
    step = max(1, -(-n // (threads * 4)))
    return [(a, min(a + step, l1)) for a in range(l0, l1, step)]


def tensor_amax(x: np.ndarray, axis: int, rotation: int = ROT_NONE, seed: int = 0,
                C: int | None = None, threads: int | None = None) -> float:
    """max |y| over the rotated tensor (rotation along the quantization axis)."""
    x = np.ascontiguousarray(x)
    dt = _as_input(x)
    R, ld = x.shape
    C = ld if C is None else C
    lines = R if axis == 1 else C
    threads = threads or default_threads()
    L = lib()

    def run(rng):
        return L.orc_tensor_amax(_ptr(x), dt, R, C, ld, axis, rotation, seed, rng[0], rng[1])

    parts = _chunks(0, lines, threads)
    if not parts:
        return 0.0
    with ThreadPoolExecutor(threads) as ex:
        return float(max(ex.map(run, parts)))


def quantize(x: np.ndarray, fmt: int, rounding: int = RTNE, rotation: int = ROT_NONE,
             axis: int = 1, double_block: bool = False, seed: int = 0, tensor_id: int = 0,
             amax: float | None = None, lines=None, C: int | None = None,
             threads: int | None = None) -> dict:
    """Quantize a row-major [R, ld] tensor (logical [R, C]) along ``axis``.

    Returns a dict with ``codes`` [L, K/2] uint8, ``scales`` [L, K/blk] uint8
    (row-major), ``outer`` [L, K/128] float32 (double block), ``tensor_scale``
    (NV/UFP4 without double block), ``amax`` and ``lines`` (the line indices).
    ``lines`` selects a subset of output lines (sampling); the tensor amax is
    always taken over the whole tensor unless ``amax`` is given.
    """
    x = np.ascontiguousarray(x)
    dt = _as_input(x)
    R, ld = x.shape
    C = ld if C is None else C
    K = C if axis == 1 else R
    nlines = R if axis == 1 else C
    blk = 32 if fmt == MXFP4 else 16
    threads = threads or default_threads()
    needs_ts = fmt in (NVFP4, UFP4) and not double_block
    if needs_ts and amax is None:
        amax = tensor_amax(x, axis, rotation, seed, C=C, threads=threads)
    ts = tensor_scale(amax, fmt) if needs_ts else 1.0
    if lines is None:
        idx = np.arange(nlines, dtype=np.int64)
    else:
        idx = np.asarray(lines, dtype=np.int64)
    n = len(idx)
    codes = np.zeros((n, K // 2), dtype=np.uint8)
    scales = np.zeros((n, K // blk), dtype=np.uint8)
    outer = np.zeros((n, max(K // 128, 0)), dtype=np.float32)
    # runs of consecutive line indices, each processed by one C call
    runs = []
    s = 0
    for t in range(1, n + 1):
        if t == n or idx[t] != idx[t - 1] + 1:
            runs.append((s, t))
            s = t
    work = []
    for (a, b) in runs:
        for (u, v) in _chunks(a, b, threads):
            work.append((u, v))
    L = lib()

    def run(uv):
        u, v = uv
        rc = L.orc_quantize_lines(_ptr(x), dt, R, C, ld, fmt, rounding, rotation, axis,
                                  int(double_block), seed, tensor_id, ts,
                                  int(idx[u]), int(idx[u]) + (v - u),
                                  _ptr(codes[u:v]), _ptr(scales[u:v]), _ptr(outer[u:v]))
        if rc:
            raise ValueError("oracle rejected the shape/format combination (code %d)" % rc)

    if work:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, work))
    return dict(codes=codes, scales=scales, outer=outer if double_block else None,
                tensor_scale=ts if needs_ts else None, amax=amax, lines=idx, K=K,
                format=fmt, double_block=bool(double_block))


def dequantize(q: dict) -> np.ndarray:
    """Exact float64 values of a quantized tensor: q * s_b * (s_t or s_o)."""
    codes = np.ascontiguousarray(q["codes"])
    scales = np.ascontiguousarray(q["scales"])
    n, K = codes.shape[0], q["K"]
    outer = q.get("outer")
    outer = np.ascontiguousarray(outer if outer is not None else np.zeros((n, 1), np.float32))
    ts = q.get("tensor_scale") or 1.0
    out = np.zeros((n, K), dtype=np.float64)
    rc = lib().orc_dequantize(_ptr(codes), _ptr(scales), _ptr(outer), ts, n, K, q["format"],
                              int(q["double_block"]), _ptr(out))
    if rc:
        raise ValueError("oracle dequantize rejected the shape (code %d)" % rc)
    return out


def dequantize32(q: dict) -> np.ndarray:
    """X^ in binary32: each exact dequantized value rounded once to nearest-even.

    "TetraJet-v2" 2.A (aligning the tensors in the backward pass: estimating
    with X^ rather than X).  The pages fix no precision for X^; the reading is
    one rounding of the exact product q * s_block * s_ref."""
    return dequantize(q).astype(np.float32)


def requantize(q: dict, fmt: int, rounding: int = RTNE, rotation: int = ROT_NONE,
               double_block: bool = False, seed: int = 0, tensor_id: int = 0,
               amax: float | None = None, lines=None, threads: int | None = None) -> dict:
    """Re-quantize the quantized tensor q ([n, K], lines along K) along the
    transposed axis: X^ = dequantize32(q), read as an [n, K] row-major tensor,
    quantized with axis 0 ("TetraJet-v2" 2.A: X^ for the backward pass, the
    transposed weight's 1x16 groups re-aligned).  The result has K lines of n
    elements; SR counters follow the [n, K] indexing of X^."""
    return quantize(dequantize32(q), fmt, rounding=rounding, rotation=rotation, axis=0,
                    double_block=double_block, seed=seed, tensor_id=tensor_id, amax=amax,
                    lines=lines, threads=threads)


def gemm(qa: dict, qb: dict):
    """C64 = deq(A) @ deq(B)^T in float64 and the bound sum_k |a_ik b_jk|.

    A is [M, K] and B is [N, K], both K-major quantized tensors (their
    lines run along K), as the Fprop / Dgrad / Wgrad GEMMs consume them.
    """
    a = dequantize(qa)
    b = dequantize(qb)
    return a @ b.T, np.abs(a) @ np.abs(b).T


# --------------------------------------------------------------------------- MXNorm

def pairwise_sum(a) -> float:
    """binary64 sum of a in index order, pairwise (halves split at the largest
    power of two below the length): the order MXNorm's block statistic uses."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    return lib().orc_pairwise_sum(_ptr(a), len(a))


def mxnorm_rho(x: np.ndarray, block: int, p: int, c: float, C: int | None = None,
               threads: int | None = None):
    """Per-row inverse-RMS estimate rho_t = c * ((1/K) sum_k m_tk^p)^(-1/p) from
    the block maxima m_tk ("MXNorm: Reusing MXFP block scales...", 2.
    Metodologia), as binary32, and each row's max |x|."""
    x = np.ascontiguousarray(x)
    dt = _as_input(x)
    R, ld = x.shape
    C = ld if C is None else C
    rho = np.zeros(R, np.float32)
    rmax = np.zeros(R, np.float32)
    threads = threads or default_threads()
    L = lib()

    def run(rng):
        a, b = rng
        rc = L.orc_mxnorm_rho(_ptr(x), dt, R, C, ld, block, p, float(c), a, b, _ptr(rho[a:b]), _ptr(rmax[a:b]))
        if rc:
            raise ValueError("oracle rejected the MXNorm shape or p (code %d)" % rc)

    parts = _chunks(0, R, threads)
    if parts:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, parts))
    return rho, rmax


def widen(x: np.ndarray) -> np.ndarray:
    """binary32 values of an oracle input (float32, or bf16 bit patterns)."""
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32)
    return np.asarray(x, dtype=np.float32)


def mxnorm(x: np.ndarray, fmt: int, p: int, c: float, rounding: int = RTNE, seed: int = 0,
           tensor_id: int = 0, C: int | None = None, lines=None) -> dict:
    """MXNorm fused with the cast: rho per row from the format's block maxima
    (32 for MXFP4, 16 for NVFP4 / UFP4), y = RN32(x * rho), and y quantized
    along the rows without rotation (the gain is folded into the next
    layer's weight, as the page does).  Returns the quantized dict of
    `quantize` with `rho` and `y` added."""
    x = np.ascontiguousarray(x)
    R, ld = x.shape
    C = ld if C is None else C
    block = 32 if fmt == MXFP4 else 16
    rho, _ = mxnorm_rho(x, block, p, c, C=C)
    y = (widen(x)[:, :C] * rho[:, None]).astype(np.float32)     # one binary32 rounding per element
    q = quantize(np.ascontiguousarray(y), fmt, rounding=rounding, rotation=ROT_NONE, axis=1, seed=seed,
                 tensor_id=tensor_id, lines=lines)
    q["rho"] = rho
    q["y"] = y
    return q


def mxnorm_constant(p: int, block: int) -> float:
    """c(p, B) for rows of i.i.d. Gaussian values: E[M^p]^(1/p) with M the
    maximum of B independent |N(0, 1)|, so that rho_t times the row's RMS
    tends to 1 (the page obtains c by Monte Carlo; here by quadrature of
    E[M^p] = int_0^inf p m^(p-1) (1 - erf(m / sqrt 2)^B) dm)."""
    from scipy import integrate, special
    f = lambda m: p * m ** (p - 1) * (1.0 - special.erf(m / np.sqrt(2.0)) ** block)
    val, _ = integrate.quad(f, 0.0, np.inf, epsabs=1e-13, epsrel=1e-12, limit=200)
    return float(val ** (1.0 / p))


# --------------------------------------------------------------------------- OutControl

def outctl_channels(x: np.ndarray, p: float) -> np.ndarray:
    """The top p of the columns (channels) of a calibration tensor by max |x|,
    ceil(p * cols) of them, ties to the lower index, in ascending order
    ("TetraJet-v2" 2.C: the channels with consistently large norms, chosen in
    a short calibration window and then kept fixed)."""
    a = np.abs(widen(np.ascontiguousarray(x))).max(axis=0)
    n = int(np.ceil(p * a.shape[0]))
    order = np.lexsort((np.arange(a.shape[0]), -a.astype(np.float64)))   # by amax descending, then index
    return np.sort(order[:n]).astype(np.int32)


def fp8_scale(amax: float) -> float:
    """The FP8 tensor scale amax / 448 in binary32 (1 if that is 0)."""
    s = np.float32(np.float32(amax) / np.float32(448.0))
    return float(s) if s > 0 else 1.0


def fp8_quantize(x: np.ndarray, K8: int, scale: float | None = None) -> dict:
    """E4M3 of the [R, n] binary32 tensor x under one tensor scale, the columns
    zero-padded to K8: codes [R, K8] (sign in bit 7), its scale and amax."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    R, n = x.shape
    amax = float(np.abs(x).max()) if x.size else 0.0
    s8 = fp8_scale(amax) if scale is None else scale
    codes = np.zeros((R, K8), np.uint8)
    if x.size:
        tmp = np.zeros((R, n), np.uint8)
        lib().orc_fp8_encode_array(_ptr(x), x.size, s8, _ptr(tmp))
        codes[:, :n] = tmp
    return dict(codes=codes, scale=s8, amax=amax, K=K8)


def fp8_dequantize(q: dict) -> np.ndarray:
    """Exact float64 values q * s8 of an FP8 tensor."""
    c = q["codes"]
    mag = np.vectorize(lambda b: lib().orc_e4m3_value(int(b) & 0x7F), otypes=[np.float64])(np.arange(256))
    sign = np.where(np.arange(256) & 0x80, -1.0, 1.0)
    table = mag * sign
    return table[c] * np.float64(q["scale"])


def outctl_quantize(x: np.ndarray, channels: np.ndarray, K8: int, fmt: int = NVFP4, rounding: int = RTNE,
                    rotation: int = ROT_NONE, seed: int = 0, tensor_id: int = 0, lines=None) -> dict:
    """OutControl's split of one operand along its channels (columns): the FP4
    part is x with the channels set to zero, quantized as `quantize` does; the
    FP8 part is x[:, channels] in E4M3 under its own tensor scale."""
    xf = widen(np.ascontiguousarray(x)).copy()
    ch = np.asarray(channels, dtype=np.int64)
    gathered = xf[:, ch].astype(np.float32)
    xf[:, ch] = 0.0
    q4 = quantize(xf, fmt, rounding=rounding, rotation=rotation, axis=1, seed=seed, tensor_id=tensor_id,
                  lines=lines)
    q8 = fp8_quantize(gathered, K8)
    if lines is not None:
        q8["codes"] = q8["codes"][np.asarray(lines)]
    return dict(fp4=q4, fp8=q8)


def gemm_outctl(a: dict, b: dict):
    """C64 = deq(A4) deq(B4)^T + deq(A8) deq(B8)^T in float64, and the bound
    sum_k |a b| over both parts."""
    C4, b4 = gemm(a["fp4"], b["fp4"])
    a8, b8 = fp8_dequantize(a["fp8"]), fp8_dequantize(b["fp8"])
    return C4 + a8 @ b8.T, b4 + np.abs(a8) @ np.abs(b8).T
