"""Parity of the rank-order reduce-scatter kernel with the CPU oracle (gpu).

Every rank's block lives on this one GPU (the kernel reads each block through
the pointer table whether it is local or a peer's mapping), and the kernel is
run once per rank -- the launches never wait on one another.  Bit-exact for
every rank's rows: the sum order is fixed by the definition.  A two-process
case maps the other process's buffer with CUDA IPC and runs the collective
wrapper end to end."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from moe_expert_epilogue_b200 import _abi, inputs, ops
from tests._util import assert_bits_equal, bits

pytestmark = pytest.mark.gpu

ODT = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}
CANARY = -3.5


def _kind(dtype):
    return "f16" if dtype == torch.float16 else "bf16"


def _place(dev, case, in_dtype, byte_offset=0, shift=None):
    """Each rank's block copied to the device at `byte_offset` inside its own
    allocation; shift = (rank, bytes) moves one rank's pointer off 16-byte
    alignment.  Returns (pointer table, keep-alive list)."""
    cap, hidden = case.buffers[0].shape
    esize = torch.empty((), dtype=in_dtype).element_size()
    keep, ptrs = [], []
    for q, b in enumerate(case.buffers):
        extra = shift[1] if shift and shift[0] == q else 0
        raw = torch.zeros(byte_offset + extra + cap * hidden * esize, dtype=torch.uint8,
                          device=dev)
        blk = raw[byte_offset + extra:].view(in_dtype).view(cap, hidden)
        blk.copy_(b.to(in_dtype).to(dev))
        keep.append(raw)
        ptrs.append(raw.data_ptr() + extra)
    return torch.tensor(ptrs, dtype=torch.int64, device=dev), keep


def _oracle(case, in_dtype, rank, out_dtype, init, ep_tokens=None, offsets=None):
    ins = [bits(b.to(in_dtype)) for b in case.buffers]
    offs = case.rank_token_offset.numpy() if offsets is None else np.asarray(offsets, np.int32)
    return oracle.ordered_reduce_scatter_v(ins, ODT[in_dtype], rank, offs,
                                           case.ep_tokens if ep_tokens is None else ep_tokens,
                                           bits(init), ODT[out_dtype])


def _run(dev, table, case, rank, in_dtype, out_dtype, init, byte_offset=0, ep_tokens=None,
         offsets=None, err=None):
    cap, hidden = case.buffers[0].shape
    offs = case.rank_token_offset if offsets is None else torch.tensor(offsets, dtype=torch.int32)
    ep = torch.tensor([case.ep_tokens if ep_tokens is None else ep_tokens], dtype=torch.int32,
                      device=dev)
    out = init.to(dev)
    ops.ordered_reduce_scatter_v(table, rank, offs.to(dev), ep, cap, hidden, in_dtype, out=out,
                                 input_byte_offset=byte_offset, dev_err=err)
    torch.cuda.synchronize()
    return out.cpu()


@pytest.mark.parametrize("world,tokens,hidden", [
    (1, 40, 64), (2, 61, 24), (3, 100, 13), (8, 300, 1032), (9, 77, 96), (17, 130, 40)])
@pytest.mark.parametrize("in_dtype,out_dtype", [
    (torch.bfloat16, torch.bfloat16), (torch.bfloat16, torch.float32),
    (torch.float16, torch.float16), (torch.float32, torch.bfloat16),
    (torch.float32, torch.float32)])
def test_reduce_scatter_bitwise_every_rank(cuda_device, world, tokens, hidden, in_dtype,
                                           out_dtype):
    case = inputs.reduce_scatter_inputs(world, tokens, hidden, spare_rows=3,
                                        sigma=4.0, seed=world * 100 + hidden)
    table, keep = _place(cuda_device, case, in_dtype)
    for rank in range(world):
        init = torch.full((case.counts[rank], hidden), CANARY, dtype=out_dtype)
        got = _run(cuda_device, table, case, rank, in_dtype, out_dtype, init)
        want, err = _oracle(case, in_dtype, rank, out_dtype, init)
        assert err == 0
        assert_bits_equal(bits(got), want, f"rank {rank}", kind=_kind(out_dtype))


@pytest.mark.parametrize("byte_offset,shift", [(16, None), (4096, None), (2, None), (0, (1, 2)),
                                               (32, (2, 8))])
def test_reduce_scatter_offsets_and_alignment(cuda_device, byte_offset, shift):
    """The block at a byte offset inside each buffer; a 2-byte offset or one
    rank's base off 16-byte alignment takes the element path -- same bits."""
    case = inputs.reduce_scatter_inputs(4, 200, 264, seed=5)
    table, keep = _place(cuda_device, case, torch.bfloat16, byte_offset, shift)
    for rank in range(4):
        init = torch.full((case.counts[rank], 264), CANARY, dtype=torch.bfloat16)
        got = _run(cuda_device, table, case, rank, torch.bfloat16, torch.bfloat16, init,
                   byte_offset=byte_offset)
        want, _ = _oracle(case, torch.bfloat16, rank, torch.bfloat16, init)
        assert_bits_equal(bits(got), want, f"rank {rank}")


def test_reduce_scatter_bad_rows(cuda_device):
    """Rows outside the data are neither read nor written and set the count
    bit; the rest are still reduced."""
    case = inputs.reduce_scatter_inputs(3, 50, 64, spare_rows=6, seed=9)
    table, keep = _place(cuda_device, case, torch.bfloat16)
    cap = 56
    init = torch.full((10, 64), CANARY, dtype=torch.float32)
    for offsets, ep in [([0, 45, 0], 50), ([0, -4, 0], 50), ([0, 40, 0], 70), ([0, 40, 0], -1)]:
        err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        got = _run(cuda_device, table, case, 1, torch.bfloat16, torch.float32, init,
                   ep_tokens=ep, offsets=offsets, err=err)
        want, oerr = _oracle(case, torch.bfloat16, 1, torch.float32, init, ep_tokens=ep,
                             offsets=offsets)
        assert int(err) == oerr == _abi.MOE_DEVERR_COUNT, (offsets, ep)
        assert np.array_equal(bits(got).view(np.uint32), want.view(np.uint32)), (offsets, ep)
    assert cap == case.buffers[0].shape[0]


def test_reduce_scatter_full_size(cuda_device):
    """8 EP ranks, 8192 tokens split raggedly, hidden 4096, bf16 partials:
    every rank's rows against the oracle."""
    case = inputs.reduce_scatter_inputs(8, 8192, 4096, seed=11)
    table, keep = _place(cuda_device, case, torch.bfloat16)
    for rank in range(8):
        init = torch.zeros((case.counts[rank], 4096), dtype=torch.bfloat16)
        got = _run(cuda_device, table, case, rank, torch.bfloat16, torch.bfloat16, init)
        want, err = _oracle(case, torch.bfloat16, rank, torch.bfloat16, init)
        assert err == 0
        assert_bits_equal(bits(got), want, f"rank {rank}")


# ------------------------------------------------------- two processes, IPC

TOK, HID, CAP = 300, 512, 304


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from moe_expert_epilogue_b200 import symmetric
        dev = torch.device("cuda", 0)
        case = inputs.reduce_scatter_inputs(world, TOK, HID, spare_rows=CAP - TOK, seed=13)
        symm = symmetric.SymmetricBuffer(256 + CAP * HID * 2, device=dev)
        symm.view(torch.bfloat16, (CAP, HID), 256).copy_(case.buffers[rank].to(dev))
        out = torch.empty(case.counts[rank], HID, dtype=torch.bfloat16, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        symmetric.ordered_reduce_scatter_v(out, symm, case.rank_token_offset.to(dev),
                                           torch.tensor([TOK], dtype=torch.int32, device=dev),
                                           CAP, HID, torch.bfloat16, input_byte_offset=256,
                                           dev_err=err)
        res = (rank, bits(out.cpu()), int(err), symm.ptrs[rank] == symm.local)
        symm.close()
        q.put(res)
    finally:
        dist.destroy_process_group()


def test_reduce_scatter_two_processes_cuda_ipc(cuda_device):
    """Two processes on this GPU: each allocates its buffer, the other maps it
    with CUDA IPC, and the collective wrapper reduces over both (host
    barriers under gloo; the kernels never wait on one another)."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=240) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    case = inputs.reduce_scatter_inputs(world, TOK, HID, spare_rows=CAP - TOK, seed=13)
    for rank, got, err, own in res:
        assert err == 0 and own
        want, _ = _oracle(case, torch.bfloat16, rank, torch.bfloat16,
                          torch.zeros(case.counts[rank], HID, dtype=torch.bfloat16))
        assert_bits_equal(got, want, f"rank {rank} over IPC")
