"""CUDA-graph capture of a whole epilogue step (gpu).

Every entry point is capturable (no allocation, no synchronisation, device-
resident counts), and the kernels are launched with programmatic stream
serialisation.  Capturing all nine launches of the benchmark step (at a small
scale) and replaying the graph must reproduce the eager results bit for bit,
also after the device-resident counts change between replays."""
import pytest
import torch

import bench
from tests._util import assert_bits_equal, bits

pytestmark = pytest.mark.gpu


def _outputs(batch):
    return {k: bits(getattr(batch, k)).copy() for k in batch.outputs}


def test_whole_step_graph_replay_matches_eager(cuda_device):
    batch = bench.Batch(cuda_device, seed=3, scale=0.02)
    kernels = batch.kernels()
    res_e0 = batch.res_e.clone()
    for k in batch.outputs:                            # rows past n_used are never written
        getattr(batch, k).zero_()
    for _, fn in kernels:
        fn()
    torch.cuda.synchronize()
    eager = _outputs(batch)
    for k in batch.outputs:
        getattr(batch, k).zero_()
    batch.res_e.copy_(res_e0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _, fn in kernels:                          # warm-up on the capture stream
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _, fn in kernels:
            fn()
    for k in batch.outputs:
        getattr(batch, k).zero_()
    batch.res_e.copy_(res_e0)
    g.replay()
    torch.cuda.synchronize()
    replayed = _outputs(batch)
    for k in batch.outputs:
        assert_bits_equal(replayed[k], eager[k], f"graph replay: {k}")
    # a smaller live prefix on the next replay: rows past it are not rewritten
    batch.act_o1.fill_(7.0)
    n_new = batch.rt.n_used // 2
    batch.n_used.fill_(n_new)
    g.replay()
    torch.cuda.synchronize()
    o = bits(batch.act_o1)
    assert_bits_equal(o[:n_new], eager["act_o1"][:n_new], "shorter n_used")
    assert (batch.act_o1[n_new:] == 7.0).all()
    del g
