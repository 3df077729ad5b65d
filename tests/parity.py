"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the CPU oracle on the same seeded inputs, and compare.

Nothing here computes the method: the GPU side is the library, the expected
side is ``oracle``; this module only moves bytes and re-indexes the tiled
scale layout documented in include/fp4.h.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

# numbering shared by the C ABI and the oracle
FMT_BLK = {0: 32, 1: 16, 2: 16}


def tiled_offsets(L: int, K: int, fmt: int) -> np.ndarray:
    """[L, K/blk] byte offsets of the tiled scale layout (include/fp4.h)."""
    blk = FMT_BLK[fmt]
    nb = K // blk
    nb4 = (nb + 3) // 4
    l = np.arange(L, dtype=np.int64)[:, None]
    b = np.arange(nb, dtype=np.int64)[None, :]
    return ((l // 128) * nb4 + b // 4) * 512 + (l % 32) * 16 + ((l % 128) // 32) * 4 + (b % 4)


def untile(buf: np.ndarray, L: int, K: int, fmt: int) -> np.ndarray:
    return buf[tiled_offsets(L, K, fmt)]


def untile_lines(buf: np.ndarray, lines: np.ndarray, K: int, fmt: int) -> np.ndarray:
    """[len(lines), K/blk] scale bytes of the given lines from a tiled buffer."""
    blk = FMT_BLK[fmt]
    nb = K // blk
    nb4 = (nb + 3) // 4
    l = np.asarray(lines, dtype=np.int64)[:, None]
    b = np.arange(nb, dtype=np.int64)[None, :]
    return buf[((l // 128) * nb4 + b // 4) * 512 + (l % 32) * 16 + ((l % 128) // 32) * 4 + (b % 4)]


def tile(rowmajor: np.ndarray, fmt: int, nbytes: int) -> np.ndarray:
    L, nb = rowmajor.shape
    K = nb * FMT_BLK[fmt]
    out = np.zeros(max(nbytes, 16), np.uint8)
    out[tiled_offsets(L, K, fmt)] = rowmajor
    return out


def oracle_input(x_cpu: torch.Tensor) -> np.ndarray:
    """The oracle's view of a CPU tensor: float32 array or bf16 bit patterns."""
    if x_cpu.dtype == torch.bfloat16:
        return x_cpu.contiguous().view(torch.int16).numpy().view(np.uint16)
    return x_cpu.contiguous().numpy()


def gpu_quantize(fp4, x_dev: torch.Tensor, cols=None, **kw) -> dict:
    q = fp4.quantize(x_dev, cols=cols, **kw)
    torch.cuda.synchronize()
    L, K, fmt = q["lines"], q["K"], q["format"]
    out = dict(codes=q["codes"].cpu().numpy(),
               scales=untile(q["scales"].cpu().numpy(), L, K, fmt) if L and K else np.zeros((L, 0), np.uint8),
               outer=q["outer"].cpu().numpy() if q["outer"] is not None else None,
               tensor_scale=float(q["tensor_scale"].cpu()[0]), raw=q)
    return out


def oracle_quantize(x_cpu: torch.Tensor, fmt, rounding=0, rotation=0, axis=1, double_block=False,
                    seed=0, tensor_id=0, amax=None, lines=None, cols=None) -> dict:
    return oracle.quantize(oracle_input(x_cpu), fmt, rounding=rounding, rotation=rotation, axis=axis,
                           double_block=double_block, seed=seed, tensor_id=tensor_id, amax=amax,
                           lines=lines, C=cols)


def assert_quant_equal(g: dict, o: dict, lines=None, what=""):
    idx = o["lines"] if lines is None else lines
    gc, gs = g["codes"][idx], g["scales"][idx]
    bad = np.argwhere(gc != o["codes"])
    assert len(bad) == 0, "%s codes differ at %d bytes, first (line, byte) %s: gpu %s oracle %s" % (
        what, len(bad), bad[:3].tolist(), gc[tuple(bad[0])], o["codes"][tuple(bad[0])])
    bad = np.argwhere(gs != o["scales"])
    assert len(bad) == 0, "%s scales differ at %d, first %s: gpu %s oracle %s" % (
        what, len(bad), bad[:3].tolist(), gs[tuple(bad[0])], o["scales"][tuple(bad[0])])
    if o["outer"] is not None:
        assert (g["outer"][idx][:, :o["outer"].shape[1]].view(np.uint32) == o["outer"].view(np.uint32)).all(), what
    if o["tensor_scale"] is not None:
        assert np.float32(g["tensor_scale"]).view(np.uint32) == np.float32(o["tensor_scale"]).view(np.uint32), (
            what, g["tensor_scale"], o["tensor_scale"])


def upload_oracle_qtensor(fp4, q: dict, device="cuda") -> dict:
    """A device qtensor holding exactly the oracle's codes and scales."""
    L, K, fmt = q["codes"].shape[0], q["K"], q["format"]
    t = dict(codes=torch.from_numpy(np.ascontiguousarray(q["codes"])).to(device),
             scales=torch.from_numpy(tile(q["scales"], fmt, fp4.fp4_scales_bytes(L, K, fmt))).to(device),
             outer=torch.from_numpy(np.ascontiguousarray(q["outer"])).to(device) if q["outer"] is not None else None,
             tensor_scale=torch.tensor([q["tensor_scale"] if q["tensor_scale"] is not None else 1.0],
                                       dtype=torch.float32, device=device),
             lines=L, K=K, format=fmt, double_block=q["double_block"])
    return t


def assert_within_gemm_bound(C: np.ndarray, C64: np.ndarray, bound: np.ndarray, bf16: bool, what=""):
    """|C - C64| <= 1e-5 * sum_k |a_ik b_jk| (+ half a bf16 ulp of the result for bf16 output)."""
    C = C.astype(np.float64)
    tol = 1e-5 * bound
    if bf16:
        mag = np.maximum(np.abs(C), np.abs(C64))
        e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
        tol = tol + np.where(mag > 0, np.exp2(e - 8), 0.0)
    err = np.abs(C - C64)
    bad = np.argwhere(err > tol)
    ratio = float((err / np.where(bound > 0, bound, 1.0)).max())
    assert len(bad) == 0, "%s: %d elements out of bound, first %s: C %r C64 %r bound %r (max err/bound %.3g)" % (
        what, len(bad), bad[:3].tolist(), C[tuple(bad[0])], C64[tuple(bad[0])], bound[tuple(bad[0])], ratio)
    return ratio


def sample_lines(n_total: int, n: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    pick = rng.choice(n_total, size=min(n, n_total), replace=False)
    return np.unique(np.concatenate([pick, [0, n_total - 1]])).astype(np.int64)
