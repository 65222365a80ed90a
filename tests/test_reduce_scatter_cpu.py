"""The multi-process side of the rank-order reduce-scatter on CPU (not gpu).

World sizes 2 and 3 over gloo, one process per rank.  A stand-in mapping
backend shares host memory between the processes (POSIX shared memory named
by the "IPC handle"), so the real exchange protocol of SymmetricBuffer runs:
allocate, export, all-gather the handles, open the peers' buffers, build the
rank-ordered pointer table, barrier, reduce, barrier, unmap, free.  The
reduction itself is the CPU oracle reading the peers' buffers through the
table, patched in for the kernel call inside the spawned CPU processes -- the
CUDA kernel itself is covered by the gpu tests.  Each rank
checks its rows bit for bit against the oracle run on all ranks' seeded
partials regenerated locally."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

CAP_SPARE, HIDDEN, TOKENS, BYTE_OFFSET = 5, 24, 61, 256


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class ShmIpc:
    """Host stand-in for the CUDA IPC backend: a pointer is a segment id in the
    high 32 bits plus a byte offset in the low ones; handles are the segments'
    names."""

    def __init__(self):
        self.segs, self.owned, self.next = {}, set(), 1
        self.log = []

    def _add(self, seg, own):
        p = self.next << 32
        self.next += 1
        self.segs[p] = seg
        if own:
            self.owned.add(p)
        return p

    def resolve(self, p):
        """(segment bytes from the pointer on, as a uint8 tensor)"""
        seg = self.segs[p & ~0xFFFFFFFF]
        off = p & 0xFFFFFFFF
        return torch.frombuffer(seg.buf, dtype=torch.uint8, count=seg.size)[off:]

    def alloc(self, nbytes):
        from multiprocessing import shared_memory
        self.log.append("alloc")
        return self._add(shared_memory.SharedMemory(create=True, size=nbytes), True)

    def export(self, p):
        name = self.segs[p].name.encode()
        return name + b"\0" * (64 - len(name))

    def open(self, handle):
        from multiprocessing import shared_memory
        self.log.append("open")
        return self._add(shared_memory.SharedMemory(name=handle.rstrip(b"\0").decode()), False)

    def close(self, p):
        self.log.append("close")
        self.segs.pop(p).close()

    def free(self, p):
        self.log.append("free")
        seg = self.segs.pop(p)
        seg.close()
        seg.unlink()

    def view(self, p, nbytes, device):
        return torch.frombuffer(self.segs[p].buf, dtype=torch.uint8, count=nbytes)

    def table(self, ptrs, device):
        return torch.tensor(ptrs, dtype=torch.int64)


def _oracle_kernel(backend):
    """Stands in for the kernel call inside the spawned CPU workers: the oracle
    reading every rank's block through the pointer table, rank order."""
    def launch(table, rank, offsets, ep_tokens, cap, hidden, in_dtype, out=None,
               input_byte_offset=0, dev_err=None):
        import oracle
        from moe_expert_epilogue_b200.inputs import bits
        ins = []
        for p in table.tolist():
            raw = backend.resolve(p)
            blk = raw[input_byte_offset:input_byte_offset + cap * hidden * 2]
            ins.append(bits(blk.view(in_dtype).view(cap, hidden).clone()))
        res, err = oracle.ordered_reduce_scatter_v(ins, oracle.BF16, rank, offsets.numpy(),
                                                   int(ep_tokens), bits(out), oracle.F32)
        assert err == 0
        out.copy_(torch.from_numpy(res))
        return out
    return launch


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from moe_expert_epilogue_b200 import inputs, ops, symmetric
        case = inputs.reduce_scatter_inputs(world, TOKENS, HIDDEN, spare_rows=CAP_SPARE, seed=7)
        cap = TOKENS + CAP_SPARE
        backend = ShmIpc()
        ops.ordered_reduce_scatter_v = _oracle_kernel(backend)     # this CPU process only
        nbytes = BYTE_OFFSET + cap * HIDDEN * 2
        symm = symmetric.SymmetricBuffer(nbytes, device=torch.device("cpu"), backend=backend)
        assert symm.ptrs[rank] == symm.local and len(symm.ptrs) == world
        symm.view(torch.bfloat16, (cap, HIDDEN), BYTE_OFFSET).copy_(case.buffers[rank])
        out = torch.full((case.counts[rank], HIDDEN), -1.0)
        symmetric.ordered_reduce_scatter_v(out, symm, case.rank_token_offset,
                                           torch.tensor([case.ep_tokens]), cap, HIDDEN,
                                           torch.bfloat16, input_byte_offset=BYTE_OFFSET)
        symm.close()
        q.put((rank, out.numpy().copy(), backend.log))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_symmetric_buffer_exchange_and_rank_order_sum(world):
    import oracle
    from moe_expert_epilogue_b200 import inputs
    from moe_expert_epilogue_b200.inputs import bits
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    case = inputs.reduce_scatter_inputs(world, TOKENS, HIDDEN, spare_rows=CAP_SPARE, seed=7)
    ins = [bits(b) for b in case.buffers]
    rows = []
    for rank, out, log in res:
        want, err = oracle.ordered_reduce_scatter_v(
            ins, oracle.BF16, rank, case.rank_token_offset.numpy(), case.ep_tokens,
            np.zeros((case.counts[rank], HIDDEN), np.float32), oracle.F32)
        assert err == 0
        assert np.array_equal(out.view(np.uint32), want.view(np.uint32)), rank
        # the mapping protocol: one allocation, world-1 peers opened, then closed, then freed
        assert log == ["alloc"] + ["open"] * (world - 1) + ["close"] * (world - 1) + ["free"]
        rows.append(out)
    # the ranks' rows tile the whole token range in order
    assert sum(r.shape[0] for r in rows) == TOKENS


def test_view_bounds():
    from moe_expert_epilogue_b200 import symmetric
    s = object.__new__(symmetric.SymmetricBuffer)
    s.nbytes, s.local, s.device, s.backend = 64, 1, torch.device("cpu"), None
    with pytest.raises(ValueError):
        s.view(torch.bfloat16, (8, 4), 2)        # 64 + 2 bytes > 64
    with pytest.raises(ValueError):
        s.view(torch.float32, (2,), 2)           # misaligned for fp32


# ------------------------------------------------------------ EP combine

EC_TOKENS, EC_TOPK, EC_EPR, EC_H = 45, 3, 4, 16


def _oracle_combine(backend):
    """Stands in for the EP-combine kernel inside the spawned CPU workers: the
    oracle reading every rank's expert rows and inverse map through the two
    pointer tables."""
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


def _combine_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from moe_expert_epilogue_b200 import inputs, ops, symmetric
        ec = inputs.ep_combine_inputs(world, EC_TOKENS, EC_TOPK, EC_EPR, 2, EC_H, seed=17)
        backend = ShmIpc()
        ops.unpermute_reduce_scatter = _oracle_combine(backend)   # this CPU process only
        cpu = torch.device("cpu")
        experts = symmetric.SymmetricBuffer(64 + ec.max_rows * EC_H * 2, device=cpu,
                                            backend=backend)
        maps = symmetric.SymmetricBuffer(EC_TOKENS * EC_EPR * 4, device=cpu, backend=backend)
        experts.view(torch.bfloat16, (ec.max_rows, EC_H), 64).copy_(ec.expert_outputs[rank])
        maps.view(torch.int32, (EC_TOKENS, EC_EPR)).copy_(ec.inverse_maps[rank])
        out = torch.zeros(ec.counts[rank], EC_H, dtype=torch.bfloat16)
        symmetric.unpermute_reduce_scatter(out, experts, maps, torch.bfloat16, ec.max_rows, EC_H,
                                           EC_EPR, EC_TOKENS, ec.rank_token_offset,
                                           torch.tensor([EC_TOKENS]), eo_byte_offset=64)
        experts.close()
        maps.close()
        q.put((rank, out.view(torch.int16).numpy().copy()))
    finally:
        dist.destroy_process_group()


def test_ep_combine_over_symmetric_buffers():
    """World size 3: each rank publishes its expert rows (at a byte offset) and
    its inverse map in two symmetric buffers; every rank's combined rows match
    the oracle run on all ranks' regenerated inputs."""
    import oracle
    from moe_expert_epilogue_b200 import inputs
    from moe_expert_epilogue_b200.inputs import bits
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_combine_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ec = inputs.ep_combine_inputs(world, EC_TOKENS, EC_TOPK, EC_EPR, 2, EC_H, seed=17)
    eos = [bits(e) for e in ec.expert_outputs]
    invs = [bits(i) for i in ec.inverse_maps]
    for rank, got in res:
        want, err = oracle.unpermute_reduce_scatter(
            eos, oracle.BF16, invs, EC_TOKENS, rank, ec.rank_token_offset.numpy(), oracle.BF16,
            np.zeros((ec.counts[rank], EC_H), np.uint16), oracle.BF16)
        assert err == 0
        assert np.array_equal(got.view(np.uint16), want), rank
