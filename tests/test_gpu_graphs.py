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


def test_next_rows_graph_replay(cuda_device):
    """The bounded SwiGLU, the fused chain and the rank-order reduce-scatter
    (one launch per rank, as the benchmark replays them) captured in one graph:
    replay equals eager, and a changed device-resident count takes effect."""
    import numpy as np
    import oracle
    from moe_expert_epilogue_b200 import inputs, ops
    d = cuda_device
    g0 = torch.Generator(device="cpu").manual_seed(5)
    y = (torch.randn(300, 256, generator=g0) * 3).to(torch.bfloat16).to(d)
    w = torch.rand(300, generator=g0).to(d)
    bound = torch.tensor([250 * 128 + 5], dtype=torch.int64, device=d)
    yo = torch.zeros(300, 128, dtype=torch.bfloat16, device=d)
    rt = inputs.routing(200, 4, 16, 8, seed=6)
    eo = inputs.expert_output_input(rt, 64, seed=7).to(d)
    pm = rt.permutation_map
    rp = torch.where(pm >= 0, rt.probs[pm.clamp(min=0).long()], torch.zeros(())).float().to(d)
    res = inputs.residual_inputs((200, 64), torch.bfloat16, seed=8, device="cpu")
    sh, rs = res["shared_expert_output"].to(d), res["residual"].to(d)
    inv, vt = rt.inverse_map.to(d), torch.tensor([200], dtype=torch.int32, device=d)
    fo = torch.zeros(200, 64, dtype=torch.bfloat16, device=d)
    case = inputs.reduce_scatter_inputs(4, 150, 64, seed=9)
    blocks = [b.to(d) for b in case.buffers]
    table = ops.pointer_table(blocks)
    offs, ep = case.rank_token_offset.to(d), torch.tensor([150], dtype=torch.int32, device=d)
    rso = [torch.zeros(c, 64, dtype=torch.bfloat16, device=d) for c in case.counts]

    def run():
        ops.weighted_silu_mul_bounded(y, w, bound, out=yo)
        ops.epilogue_fused(eo, rp, inv, vt, sh, rs, out=fo)
        for r in range(4):
            ops.ordered_reduce_scatter_v(table, r, offs, ep, 150, 64, torch.bfloat16, out=rso[r])

    run()
    torch.cuda.synchronize()
    eager = [bits(t).copy() for t in [yo, fo] + rso]
    for t in [yo, fo] + rso:
        t.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for t in [yo, fo] + rso:
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    g.replay()
    torch.cuda.synchronize()
    for i, t in enumerate([yo, fo] + rso):
        assert_bits_equal(bits(t), eager[i], f"graph replay output {i}")
    # the rank-order sums against the oracle too
    ins = [bits(b) for b in case.buffers]
    for r in range(4):
        want, err = oracle.ordered_reduce_scatter_v(ins, oracle.BF16, r,
                                                    case.rank_token_offset.numpy(), 150,
                                                    np.zeros((case.counts[r], 64), np.uint16),
                                                    oracle.BF16)
        assert err == 0
        assert_bits_equal(bits(rso[r]), want, f"rank {r}")
    # a smaller device-resident bound on the next replay
    yo.fill_(2.0)
    bound.fill_(100 * 128)
    g.replay()
    torch.cuda.synchronize()
    assert_bits_equal(bits(yo)[:100], eager[0][:100], "shorter bound")
    assert (yo[100:] == 2.0).all()
    del g
