"""The multi-GPU leg of bench.py on CPU (not gpu): `measure_collectives` over
a gloo process group of two ranks.

Each rank runs the leg exactly as a GPU rank would -- symmetric buffers
allocated, exported, all-gathered and opened, the two collectives called
through `symmetric` between their stream barriers, kernel and whole-call times
taken around the launch hooks and maxed over the ranks -- with the host
stand-in for the CUDA IPC mapping and the CPU oracle patched in for the two
kernels inside the spawned workers.  Every rank's outputs are then checked
bit for bit against the oracle run here on the regenerated inputs."""
import os

import numpy as np
import torch
import torch.multiprocessing as mp

from tests.test_reduce_scatter_cpu import ShmIpc, _free_port

TOKENS, HIDDEN, TOPK, EPR, SEED = 61, 24, 3, 4, 1000


def _rs_standin(backend):
    def launch(table, rank, offsets, ep_tokens, cap, hidden, in_dtype, out=None,
               input_byte_offset=0, dev_err=None):
        import oracle
        from moe_expert_epilogue_b200.inputs import bits
        ins = [bits(backend.resolve(p)[input_byte_offset:input_byte_offset + cap * hidden * 2]
                    .view(in_dtype).view(cap, hidden).clone()) for p in table.tolist()]
        res, err = oracle.ordered_reduce_scatter_v(ins, oracle.BF16, rank, offsets.numpy(),
                                                   int(ep_tokens), bits(out), oracle.BF16)
        assert err == 0
        out.view(torch.int16).copy_(torch.from_numpy(res.view(np.int16)))
        return out
    return launch


def _combine_standin(backend):
    def launch(eo_t, eo_dtype, max_rows, inv_t, E, cap, ep_tokens, rank, offsets, hidden,
               out=None, partial_dtype=None, dev_err=None):
        import oracle
        from moe_expert_epilogue_b200.inputs import bits
        eos = [bits(backend.resolve(p)[:max_rows * hidden * 2].view(eo_dtype)
                    .view(max_rows, hidden).clone()) for p in eo_t.tolist()]
        invs = [backend.resolve(p)[:cap * E * 4].view(torch.int32).view(cap, E).numpy().copy()
                for p in inv_t.tolist()]
        res, err = oracle.unpermute_reduce_scatter(eos, oracle.BF16, invs, int(ep_tokens), rank,
                                                   offsets.numpy(), oracle.BF16, bits(out),
                                                   oracle.BF16)
        assert err == 0
        out.view(torch.int16).copy_(torch.from_numpy(res.view(np.int16)))
        return out
    return launch


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from moe_expert_epilogue_b200 import ops
        backend = ShmIpc()
        ops.ordered_reduce_scatter_v = _rs_standin(backend)     # this CPU process only
        ops.unpermute_reduce_scatter = _combine_standin(backend)
        stats, outs = bench.measure_collectives(
            torch.device("cpu"), SEED, 2, tokens=TOKENS, hidden=HIDDEN, top_k=TOPK,
            experts_per_rank=EPR, backend=backend, return_outputs=True)
        q.put((rank, stats, {k: v.view(torch.int16).numpy().copy() for k, v in outs.items()},
               backend.log))
    finally:
        dist.destroy_process_group()


def test_bench_collectives_leg_over_gloo():
    import oracle
    from moe_expert_epilogue_b200 import inputs
    from moe_expert_epilogue_b200.inputs import bits
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    case = inputs.reduce_scatter_inputs(world, TOKENS, HIDDEN, seed=SEED + 8)
    ec = inputs.ep_combine_inputs(world, TOKENS, TOPK, EPR, 128, HIDDEN, seed=SEED + 9)
    ins = [bits(b) for b in case.buffers]
    eos = [bits(e) for e in ec.expert_outputs]
    invs = [bits(i) for i in ec.inverse_maps]
    kernel_times = set()
    for rank, stats, outs, log in res:
        want, err = oracle.ordered_reduce_scatter_v(
            ins, oracle.BF16, rank, case.rank_token_offset.numpy(), case.ep_tokens,
            np.zeros((case.counts[rank], HIDDEN), np.uint16), oracle.BF16)
        assert err == 0
        assert np.array_equal(outs["ordered_reduce_scatter_v"].view(np.uint16), want), rank
        want, err = oracle.unpermute_reduce_scatter(
            eos, oracle.BF16, invs, TOKENS, rank, ec.rank_token_offset.numpy(), oracle.BF16,
            np.zeros((ec.counts[rank], HIDDEN), np.uint16), oracle.BF16)
        assert err == 0
        assert np.array_equal(outs["unpermute_reduce_scatter"].view(np.uint16), want), rank
        # three symmetric buffers (reduce-scatter blocks, expert rows, inverse maps),
        # each opened from the one peer, then unmapped and freed
        assert log.count("alloc") == 3 and log.count("open") == 3
        assert log.count("close") == 3 and log.count("free") == 3
        assert stats["world"] == world
        for name in ("ordered_reduce_scatter_v", "unpermute_reduce_scatter"):
            s = stats[name]
            assert s["kernel_us"] > 0 and s["call_us"] >= s["kernel_us"]
            assert s["nvlink_bytes"] > 0 and s["bytes_read_written"] > s["nvlink_bytes"]
            kernel_times.add((name, s["kernel_us"], s["call_us"]))
    # the times are maxed over the ranks: both ranks report the same numbers
    assert len(kernel_times) == 2
    # NVLink bytes of the reduce-scatter: this rank's rows of the one peer's block
    for rank, stats, _, _ in res:
        assert stats["ordered_reduce_scatter_v"]["nvlink_bytes"] == \
            case.counts[rank] * HIDDEN * 2 * (world - 1)
