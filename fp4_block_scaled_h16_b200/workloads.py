"""Seeded synthetic inputs shaped like the pages' Llama-3.1-8B workloads.

This module only draws random tensors; it holds none of the quantization or
GEMM arithmetic, so the CUDA path and the CPU oracle can both take their
inputs from it.  Every generator is numpy PCG64 (``default_rng(seed)``) with
a fixed draw order; float32 draws are rounded to bfloat16 by torch's
round-to-nearest-even cast where a workload is bf16.

Shapes follow Llama-3.1-8B linears (hidden 4096, 32 query / 8 key-value heads
of 128, FFN 14336) at 8192 tokens, the model the MXFP4 pretraining page trains
("Pre-addestramento di Modelli Linguistici di Grandi Dimensioni con MXFP4",
Metodologia).  Activations carry a few outlier channels ("TetraJet-v2",
section 1: a few activation channels with huge magnitudes); gradients are
heavy-tailed (Laplace); weights are N(0, 0.02).
"""
from __future__ import annotations

import numpy as np
import torch

HIDDEN, QKV_OUT, FFN, TOKENS = 4096, 6144, 14336, 8192


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a CPU bfloat16 tensor (the oracle's bf16 input form)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def normal(rng, shape, std=1.0):
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(std)


def activations_with_outliers(rng, rows, cols, n_outliers=8, factor=64.0):
    """N(0,1) activations with ``n_outliers`` seeded channels (columns) scaled up."""
    x = normal(rng, (rows, cols))
    ch = rng.choice(cols, min(n_outliers, cols), replace=False)
    x[:, ch] *= np.float32(factor)
    return x


def laplace_grad(rng, rows, cols, scale=1e-3):
    return rng.laplace(0.0, scale, (rows, cols)).astype(np.float32)


def swiglu_hidden(rng, rows, cols):
    """H = a * silu(b), a, b independent N(0,1): the down projection's input."""
    a = normal(rng, (rows, cols))
    b = normal(rng, (rows, cols))
    return a * (b / (np.float32(1.0) + np.exp(-b)))


# ----------------------------------------------------------------------- workloads

def tiny_mxfp4(seed=0, M=256, N=256, K=512):
    """A fp32 [M, K] and B fp32 [K, N], both N(0, 1), drawn A then B."""
    rng = np.random.default_rng(seed)
    return dict(A=torch.from_numpy(normal(rng, (M, K))), B=torch.from_numpy(normal(rng, (K, N))))


def nvfp4_fprop_qkv(seed=0, T=TOKENS, d_in=HIDDEN, d_out=QKV_OUT, n_outliers=8):
    """Fprop of the QKV projection: X bf16 [T, d_in] with outlier channels, W bf16 [d_out, d_in]."""
    rng = np.random.default_rng(seed)
    X = activations_with_outliers(rng, T, d_in, n_outliers)
    W = normal(rng, (d_out, d_in), 0.02)
    return dict(X=_bf16(X), W=_bf16(W))


def mxfp4_wgrad_down(seed=0, T=TOKENS, d_model=HIDDEN, d_ffn=FFN):
    """Wgrad of the down projection: dY bf16 [T, d_model] Laplace(0, 1e-3), H bf16 [T, d_ffn]."""
    rng = np.random.default_rng(seed)
    dY = laplace_grad(rng, T, d_model)
    H = swiglu_hidden(rng, T, d_ffn)
    return dict(dY=_bf16(dY), H=_bf16(H))


def nvfp4_dgrad_down(seed=0, T=TOKENS, d_model=HIDDEN, d_ffn=FFN):
    """Dgrad of the down projection: dY bf16 [T, d_model], Wd bf16 [d_model, d_ffn] N(0, 0.02)."""
    rng = np.random.default_rng(seed)
    dY = laplace_grad(rng, T, d_model)
    Wd = normal(rng, (d_model, d_ffn), 0.02)
    return dict(dY=_bf16(dY), Wd=_bf16(Wd))


# Llama-3.1-8B decoder-layer linears: (name, d_in, d_out, input recipe)
LAYER_LINEARS = (
    ("qkv", HIDDEN, QKV_OUT, "act"),
    ("o", HIDDEN, HIDDEN, "act"),
    ("gate_up", HIDDEN, 2 * FFN, "act"),
    ("down", FFN, HIDDEN, "swiglu"),
)


def layer_linear(name, seed=0, T=TOKENS, scale_dims=1):
    """Inputs of one linear of the layer: X [T, d_in], W [d_out, d_in], dY [T, d_out].

    ``scale_dims`` divides d_in, d_out and T for small test versions of the
    same recipe.
    """
    index = [n for n, _, _, _ in LAYER_LINEARS].index(name)
    _, d_in, d_out, recipe = LAYER_LINEARS[index]
    d_in, d_out, T = d_in // scale_dims, d_out // scale_dims, T // scale_dims
    rng = np.random.default_rng([seed, index])
    X = activations_with_outliers(rng, T, d_in) if recipe == "act" else swiglu_hidden(rng, T, d_in)
    W = normal(rng, (d_out, d_in), 0.02)
    dY = laplace_grad(rng, T, d_out)
    return dict(X=_bf16(X), W=_bf16(W), dY=_bf16(dY))


# The six quantized operands of one linear, in role order: (tensor, axis,
# stochastic rounding).  Fprop Y = X W^T takes X and W along their rows
# (axis 1); Dgrad dX = dY W takes dY along its rows and W along its columns
# (axis 0); Wgrad dW = dY^T X takes dY and X along their columns (axis 0),
# with stochastic rounding ("Pre-addestramento ... con MXFP4", Metodologia:
# the three GEMMs of every linear).
LAYER_OPERANDS = (("X", 1, False), ("W", 1, False), ("dY", 1, False),
                  ("W", 0, False), ("dY", 0, True), ("X", 0, True))
# The three GEMMs: (name, operand role of A, operand role of B, bf16 output?)
LAYER_GEMMS = (("fprop", 0, 1, True), ("dgrad", 2, 3, True), ("wgrad", 4, 5, False))


def layer_tensor_id(linear_index: int, role: int) -> int:
    """Stochastic-rounding stream of one operand: 16 * linear + role."""
    return 16 * linear_index + role
