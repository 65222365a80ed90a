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
    """Host stand-in for the CUDA IPC backend: pointers are ids of shared-memory
    segments, handles are the segments' names."""

    def __init__(self):
        self.segs, self.owned, self.next = {}, set(), 1
        self.log = []

    def _add(self, seg, own):
        p = self.next
        self.next += 1
        self.segs[p] = seg
        if own:
            self.owned.add(p)
        return p

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
            raw = backend.view(p, backend.segs[p].size, None)
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
