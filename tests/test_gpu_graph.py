"""The hot path inside a CUDA graph: one Fprop step (quantize X and W with
their tensor amax computed in one cooperative launch each, then the NVFP4
GEMM) is captured once and replayed; every replay must give the bits of the
eager step, also after the inputs change in place."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp4(cuda_device):
    from fp4_block_scaled_h16_b200 import fp4 as m
    return m


def test_fprop_step_replays_from_a_cuda_graph(fp4):
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(0)
    M, N, K = 512, 768, 1024
    X = torch.randn((M, K), generator=g).to(torch.bfloat16).to(dev)
    W = (torch.randn((N, K), generator=g) * 0.02).to(torch.bfloat16).to(dev)
    qx = fp4.alloc_qtensor(M, K, fp4.FP4_NVFP4, device=dev)
    qw = fp4.alloc_qtensor(N, K, fp4.FP4_NVFP4, device=dev)
    wsx = torch.empty(256, dtype=torch.uint8, device=dev)
    wsw = torch.empty(256, dtype=torch.uint8, device=dev)
    C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def step():
        fp4.quantize(X, fp4.FP4_NVFP4, rotation=fp4.FP4_ROT_H16, out=qx, workspace=wsx)
        fp4.quantize(W, fp4.FP4_NVFP4, rotation=fp4.FP4_ROT_H16, out=qw, workspace=wsw)
        fp4.gemm(qx, qw, fp4.FP4_OUT_BF16, out=C)

    step()
    torch.cuda.synchronize()
    eager = C.clone()
    assert fp4.fp4_last_error() == fp4.FP4_OK

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        step()                                    # warm-up on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)

    C.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(C.view(torch.int16), eager.view(torch.int16))

    X.mul_(-2.0)                                  # new inputs in place: the graph reads them
    graph.replay()
    torch.cuda.synchronize()
    replayed = C.clone()
    step()
    torch.cuda.synchronize()
    assert torch.equal(replayed.view(torch.int16), C.view(torch.int16))
    assert not torch.equal(replayed.view(torch.int16), eager.view(torch.int16))
    assert fp4.fp4_last_error() == fp4.FP4_OK
    del graph
