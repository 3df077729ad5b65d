"""World-size-2 tests of the multi-rank host logic on CPU (gloo backend).

The CUDA calls are stood in for by the oracle on CPU: each rank takes the amax
of its row shard, the ranks take the max over ranks (the same helper the
library path uses), and each quantizes its rows with that amax.  The result
must equal the unsharded quantization row for row.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from fp4_block_scaled_h16_b200.dist import global_amax_, max_over_ranks
        rng = np.random.default_rng(0)
        x = rng.standard_normal((64, 256)).astype(np.float32)
        x[rng.integers(64), rng.integers(256)] = 40.0
        shard = x[rank * 32:(rank + 1) * 32]
        local = torch.tensor([oracle.tensor_amax(shard, 1, oracle.ROT_H16)], dtype=torch.float32)
        global_amax_(local)
        q = oracle.quantize(shard, oracle.NVFP4, rotation=oracle.ROT_H16, amax=float(local[0]))
        full = oracle.quantize(x, oracle.NVFP4, rotation=oracle.ROT_H16)
        ok = (q["codes"] == full["codes"][rank * 32:(rank + 1) * 32]).all() and \
             (q["scales"] == full["scales"][rank * 32:(rank + 1) * 32]).all() and \
             q["tensor_scale"] == full["tensor_scale"]
        t = max_over_ranks([1.0 + rank, 5.0 - rank])
        out[rank] = int(bool(ok) and t == [2.0, 5.0] and float(local[0]) == full["amax"])
    finally:
        dist.destroy_process_group()


def test_sharded_amax_quantization_equals_unsharded():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert dict(out) == {0: 1, 1: 1}


class _FakeFp4:
    """Stands in for the binding in a host-logic test: only the constants."""
    FP4_RTNE, FP4_SR = 0, 1


def test_row_shard_helper_refuses_stochastic_rounding():
    # the SR counter of a shard is shard-local, so sharded SR is not the
    # unsharded result; the helper must say so before launching anything
    from fp4_block_scaled_h16_b200.dist import quantize_row_shard
    with pytest.raises(ValueError, match="stochastic rounding"):
        quantize_row_shard(_FakeFp4, torch.zeros((4, 16)), fmt=1, rounding=_FakeFp4.FP4_SR)
