"""Multi-GPU plumbing (torch.distributed, one process per GPU).

The hot path shards by independent problems -- every rank quantizes and
multiplies its own operands -- so the data path needs no collective.  The one
exchange the method has appears when the rows of a single NVFP4 / UFP4 tensor
are spread over ranks: the tensor scale amax / (Q * 448) needs the amax of the
whole rotated tensor ("TetraJet-v2" 2.A names this tensor-wide amax as what
the double block avoids).  Each rank then runs fp4_amax on its shard, the
ranks take the max of one float, and each quantizes its shard with
fp4_quantize(tensor_amax=...).  Under round-to-nearest-even that is exactly
the unsharded result.  Stochastic rounding is refused here: its Philox counter
is the element index within the tensor the call sees, i.e. the shard, so
every rank would draw the same words as rank 0 instead of those of its rows
of the whole tensor.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def global_amax_(local_amax: torch.Tensor, group=None) -> torch.Tensor:
    """In-place max over ranks of a one-element amax tensor."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(local_amax, op=dist.ReduceOp.MAX, group=group)
    return local_amax


def quantize_row_shard(fp4, x_shard: torch.Tensor, fmt: int, rounding: int = 0, rotation: int = 0,
                       seed: int = 0, tensor_id: int = 0, group=None) -> dict:
    """Quantize this rank's rows of a tensor along axis 1 with the tensor scale
    of the whole (sharded) tensor: local amax, max all-reduce, quantize.
    Round-to-nearest-even only (see the module docstring): ``rounding`` other
    than RTNE raises ValueError before anything is launched."""
    if rounding != fp4.FP4_RTNE:
        raise ValueError("quantize_row_shard: stochastic rounding of a row shard would not draw the "
                         "unsharded tensor's random words (the counter is the shard-local index)")
    amax = torch.empty(1, dtype=torch.float32, device=x_shard.device)
    rows, cols = x_shard.shape
    fp4.fp4_amax(x_shard, fp4.in_dtype_of(x_shard), rows, cols, x_shard.stride(0) if rows > 1 else cols,
                 rotation, 1, seed, amax)
    global_amax_(amax, group)
    return fp4.quantize(x_shard, fmt, rounding, rotation, axis=1, seed=seed, tensor_id=tensor_id,
                        tensor_amax=amax)


def max_over_ranks(values, device=None, group=None) -> list:
    """Element-wise max over ranks of a list of floats (timings)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return [float(v) for v in t.cpu()]
