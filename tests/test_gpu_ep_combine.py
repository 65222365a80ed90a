"""Parity of the EP-combine kernel (every rank's unpermute and the rank-order
reduce-scatter in one kernel) with the CPU oracle and with the two library
kernels it fuses (gpu).

Every rank's expert rows and inverse map live on this one GPU; the kernel
reads them through the pointer tables exactly as it reads peers' memory, and
runs once per rank (the launches never wait on one another).  Bit-exact: the
sum orders (experts ascending within a rank, ranks ascending) and the
rounding of each rank's partial are fixed by the definition."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_epilogue_b200 import _abi, inputs, ops
from tests._util import assert_bits_equal, bits

pytestmark = pytest.mark.gpu

ODT = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}
KIND = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "bf16"}


def _tables(dev, case, shift=None):
    """Device copies of every rank's expert rows and inverse map, and their
    pointer tables; shift = (rank, bytes) moves one rank's expert rows off
    16-byte alignment."""
    keep, eo_ptrs, inv_ptrs = [], [], []
    for q, (eo, inv) in enumerate(zip(case.expert_outputs, case.inverse_maps)):
        extra = shift[1] if shift and shift[0] == q else 0
        raw = torch.zeros(extra + eo.numel() * eo.element_size(), dtype=torch.uint8, device=dev)
        blk = raw[extra:].view(eo.dtype).view(eo.shape)
        blk.copy_(eo.to(dev))
        inv_d = inv.to(dev)
        keep += [raw, inv_d]
        eo_ptrs.append(raw.data_ptr() + extra)
        inv_ptrs.append(inv_d.data_ptr())
    return (torch.tensor(eo_ptrs, dtype=torch.int64, device=dev),
            torch.tensor(inv_ptrs, dtype=torch.int64, device=dev), keep)


def _run(dev, case, eo_t, inv_t, rank, out_dtype, partial_dtype, init, ep_tokens=None,
         offsets=None, err=None):
    E = case.inverse_maps[0].shape[1]
    hidden = case.expert_outputs[0].shape[1]
    offs = case.rank_token_offset if offsets is None else torch.tensor(offsets, dtype=torch.int32)
    ep = torch.tensor([case.tokens if ep_tokens is None else ep_tokens], dtype=torch.int32,
                      device=dev)
    out = init.to(dev)
    ops.unpermute_reduce_scatter(eo_t, case.expert_outputs[0].dtype, case.max_rows, inv_t, E,
                                 case.tokens, ep, rank, offs.to(dev), hidden, out=out,
                                 partial_dtype=partial_dtype, dev_err=err)
    torch.cuda.synchronize()
    return out.cpu()


def _oracle(case, rank, out_dtype, partial_dtype, init, ep_tokens=None, offsets=None):
    eo_dt = case.expert_outputs[0].dtype
    offs = case.rank_token_offset.numpy() if offsets is None else np.asarray(offsets, np.int32)
    return oracle.unpermute_reduce_scatter(
        [bits(e) for e in case.expert_outputs], ODT[eo_dt], [bits(i) for i in case.inverse_maps],
        case.tokens if ep_tokens is None else ep_tokens, rank, offs, ODT[partial_dtype],
        bits(init), ODT[out_dtype])


CASES = [  # world, tokens, top_k, experts per rank, align, hidden
    (1, 40, 4, 8, 4, 64), (2, 61, 2, 4, 4, 24), (4, 200, 8, 16, 16, 1032),
    (8, 300, 8, 8, 128, 512), (3, 50, 3, 5, 2, 13), (9, 77, 4, 2, 8, 96), (17, 64, 4, 1, 4, 40),
    (2, 40, 8, 64, 4, 64)]
DTYPES = [  # expert outputs, partial blocks, output
    (torch.bfloat16, torch.bfloat16, torch.bfloat16), (torch.bfloat16, torch.float32, torch.bfloat16),
    (torch.bfloat16, torch.float32, torch.float32), (torch.float16, torch.float16, torch.float32),
    (torch.float32, torch.float32, torch.float32)]


@pytest.mark.parametrize("world,tokens,top_k,epr,align,hidden", CASES)
@pytest.mark.parametrize("eo_dtype,partial_dtype,out_dtype", DTYPES)
def test_ep_combine_bitwise_every_rank(cuda_device, world, tokens, top_k, epr, align, hidden,
                                       eo_dtype, partial_dtype, out_dtype):
    case = inputs.ep_combine_inputs(world, tokens, top_k, epr, align, hidden, dtype=eo_dtype,
                                    seed=world * 1000 + hidden)
    eo_t, inv_t, keep = _tables(cuda_device, case)
    for rank in range(world):
        init = torch.full((case.counts[rank], hidden), -2.5, dtype=out_dtype)
        got = _run(cuda_device, case, eo_t, inv_t, rank, out_dtype, partial_dtype, init)
        want, err = _oracle(case, rank, out_dtype, partial_dtype, init)
        assert err == 0
        assert_bits_equal(bits(got), want, f"rank {rank}", kind=KIND[out_dtype])


# Shapes aimed at the TMA-staged kernel (up to 64 (rank, local expert) pairs,
# hidden % 8 == 0): lists longer than one stage of 8 rows, rows cut into chunks
# of 2048 columns with a ragged last chunk, a one-unit row; and one shape past
# 64 pairs, which takes the register-staged kernel.
CASES_TMA = [  # world, tokens, top_k, experts per rank, align, hidden
    (2, 50, 20, 16, 4, 264), (4, 100, 12, 16, 8, 4104), (8, 64, 8, 8, 16, 7168),
    (1, 33, 1, 1, 1, 8), (9, 60, 4, 8, 8, 96)]


@pytest.mark.parametrize("world,tokens,top_k,epr,align,hidden", CASES_TMA)
@pytest.mark.parametrize("eo_dtype,partial_dtype,out_dtype", DTYPES)
def test_ep_combine_stages_and_chunks(cuda_device, world, tokens, top_k, epr, align, hidden,
                                      eo_dtype, partial_dtype, out_dtype):
    case = inputs.ep_combine_inputs(world, tokens, top_k, epr, align, hidden, dtype=eo_dtype,
                                    seed=world * 77 + hidden)
    eo_t, inv_t, keep = _tables(cuda_device, case)
    _abi.moe_device_errors(clear=True)
    for rank in range(world):
        init = torch.full((case.counts[rank], hidden), -2.5, dtype=out_dtype)
        got = _run(cuda_device, case, eo_t, inv_t, rank, out_dtype, partial_dtype, init)
        want, err = _oracle(case, rank, out_dtype, partial_dtype, init)
        assert err == 0
        assert_bits_equal(bits(got), want, f"rank {rank}", kind=KIND[out_dtype])
    assert _abi.moe_device_errors(clear=True) == 0


def test_ep_combine_tokens_without_rows(cuda_device):
    """Tokens none of whose experts any rank holds (all inverse entries < 0)
    get the empty rank-order sum, +0, like their all-zero partial block rows;
    the tokens around them are unaffected."""
    case = inputs.ep_combine_inputs(4, 90, 4, 4, 8, 2056, seed=12)
    for q in range(4):
        inv = case.inverse_maps[q].clone()
        inv[::7] = -1
        inv[40:44] = -1
        case.inverse_maps[q] = inv
    eo_t, inv_t, keep = _tables(cuda_device, case)
    for rank in range(4):
        init = torch.full((case.counts[rank], 2056), 9.0, dtype=torch.bfloat16)
        got = _run(cuda_device, case, eo_t, inv_t, rank, torch.bfloat16, torch.bfloat16, init)
        want, err = _oracle(case, rank, torch.bfloat16, torch.bfloat16, init)
        assert err == 0
        assert_bits_equal(bits(got), want, f"rank {rank}")


@pytest.mark.parametrize("partial_dtype", [torch.bfloat16, torch.float32])
def test_ep_combine_subnormal_and_signed_zero_rows(cuda_device, partial_dtype):
    """Expert rows of bf16 subnormals, signed zeros and their negations: the
    packed adds keep subnormal operands and sums (no flush to zero), and a
    one-row partial of -0 still becomes +0 + -0 = +0 as in the two steps."""
    case = inputs.ep_combine_inputs(2, 64, 4, 4, 8, 4096, seed=21)
    g = torch.Generator().manual_seed(22)
    for q in range(2):
        eo = case.expert_outputs[q]
        raw = torch.randint(1, 0x80, eo.shape, generator=g, dtype=torch.int32)  # subnormal bits
        sign = torch.randint(0, 2, eo.shape, generator=g, dtype=torch.int32) << 15
        bits16 = (raw | sign).to(torch.int16)
        bits16[:, ::97] = 0
        bits16[:, 1::97] = -32768                                              # -0.0
        case.expert_outputs[q] = bits16.view(torch.bfloat16)
    eo_t, inv_t, keep = _tables(cuda_device, case)
    for rank in range(2):
        init = torch.zeros(case.counts[rank], 4096, dtype=torch.float32)
        got = _run(cuda_device, case, eo_t, inv_t, rank, torch.float32, partial_dtype, init)
        want, err = _oracle(case, rank, torch.float32, partial_dtype, init)
        assert err == 0
        assert np.array_equal(bits(got).view(np.uint32), want.view(np.uint32)), rank
        assert (bits(got) != 0).any() and np.isfinite(bits(got)).all()


def _two_step(dev, case, rank, partial_dtype, out_dtype):
    """The pages' form with the library's own kernels: each rank's unpermute
    into a partial block, then the reduce-scatter of the blocks."""
    hidden = case.expert_outputs[0].shape[1]
    blocks = []
    vt = torch.tensor([case.tokens], dtype=torch.int32, device=dev)
    for eo, inv in zip(case.expert_outputs, case.inverse_maps):
        blk = torch.zeros(case.tokens, hidden, dtype=partial_dtype, device=dev)
        ops.unpermute_ordered(eo.to(dev), inv.to(dev), vt, blk)
        blocks.append(blk)
    out = torch.zeros(case.counts[rank], hidden, dtype=out_dtype, device=dev)
    ops.ordered_reduce_scatter_v(ops.pointer_table(blocks), rank, case.rank_token_offset.to(dev),
                                 vt, case.tokens, hidden, partial_dtype, out=out)
    torch.cuda.synchronize()
    return out.cpu()


@pytest.mark.parametrize("partial_dtype,out_dtype", [(torch.bfloat16, torch.bfloat16),
                                                     (torch.float32, torch.bfloat16)])
def test_ep_combine_equals_unpermute_then_reduce_scatter(cuda_device, partial_dtype, out_dtype):
    """8 EP ranks, 8192 tokens, top-8 of 64 experts (8 per rank), hidden 4096:
    the fused kernel gives the bits of the two library kernels it replaces,
    for every rank's rows."""
    case = inputs.ep_combine_inputs(8, 8192, 8, 8, 128, 4096, seed=3, device="cpu")
    eo_t, inv_t, keep = _tables(cuda_device, case)
    for rank in range(8):
        init = torch.zeros(case.counts[rank], 4096, dtype=out_dtype)
        got = _run(cuda_device, case, eo_t, inv_t, rank, out_dtype, partial_dtype, init)
        assert_bits_equal(bits(got), bits(_two_step(cuda_device, case, rank, partial_dtype,
                                                    out_dtype)), f"rank {rank}")


@pytest.mark.parametrize("shift", [(0, 2), (2, 8)])
def test_ep_combine_unaligned_rows(cuda_device, shift):
    case = inputs.ep_combine_inputs(4, 120, 4, 4, 8, 264, seed=5)
    eo_t, inv_t, keep = _tables(cuda_device, case, shift)
    for rank in range(4):
        init = torch.zeros(case.counts[rank], 264, dtype=torch.bfloat16)
        got = _run(cuda_device, case, eo_t, inv_t, rank, torch.bfloat16, torch.bfloat16, init)
        want, _ = _oracle(case, rank, torch.bfloat16, torch.bfloat16, init)
        assert_bits_equal(bits(got), want, f"rank {rank}")


def test_ep_combine_bad_rows_and_entries(cuda_device):
    case = inputs.ep_combine_inputs(3, 60, 3, 4, 4, 32, seed=6)
    init = torch.full((10, 32), 7.0)
    eo_t, inv_t, keep = _tables(cuda_device, case)
    for offsets, ep in [([0, 55, 0], 60), ([0, -3, 0], 60), ([0, 50, 0], 80)]:
        err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        got = _run(cuda_device, case, eo_t, inv_t, 1, torch.float32, torch.float32, init,
                   ep_tokens=ep, offsets=offsets, err=err)
        want, oerr = _oracle(case, 1, torch.float32, torch.float32, init, ep_tokens=ep,
                             offsets=offsets)
        assert int(err) == _abi.MOE_DEVERR_COUNT and oerr & _abi.MOE_DEVERR_COUNT
        assert np.array_equal(bits(got).view(np.uint32), want.view(np.uint32)), (offsets, ep)
    # an inverse-map entry past the expert rows, in rank 1's own tokens: skipped, reported
    bad = case.inverse_maps[2].clone()
    t = int(case.rank_token_offset[1])
    e = int(torch.nonzero(bad[t] >= 0)[0, 0]) if (bad[t] >= 0).any() else 0
    bad[t, e] = case.max_rows + 5
    case.inverse_maps[2] = bad
    eo_t, inv_t, keep = _tables(cuda_device, case)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    init = torch.zeros(case.counts[1], 32)
    got = _run(cuda_device, case, eo_t, inv_t, 1, torch.float32, torch.float32, init, err=err)
    want, oerr = _oracle(case, 1, torch.float32, torch.float32, init)
    assert int(err) == _abi.MOE_DEVERR_INVERSE and oerr == _abi.MOE_DEVERR_INVERSE
    assert np.array_equal(bits(got).view(np.uint32), want.view(np.uint32))


def test_ep_combine_long_launch(cuda_device):
    """A launch with many items per warp takes the 4-rows-in-flight kernel:
    2 ranks, 40000 tokens (about 20000 a rank) x top-4 of 8 experts, hidden
    4096 -- still the two library kernels' bits for every row."""
    case = inputs.ep_combine_inputs(2, 40000, 4, 4, 128, 4096, seed=8, device=cuda_device)
    eo_t, inv_t, keep = _tables(cuda_device, case)
    for rank in range(2):
        init = torch.zeros(case.counts[rank], 4096, dtype=torch.bfloat16)
        got = _run(cuda_device, case, eo_t, inv_t, rank, torch.bfloat16, torch.bfloat16, init)
        assert_bits_equal(bits(got), bits(_two_step(cuda_device, case, rank, torch.bfloat16,
                                                    torch.bfloat16)), f"rank {rank}")


# ------------------------------------------------------- two processes, IPC

def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_worker(rank, world, port, q):
    import os
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from moe_expert_epilogue_b200 import symmetric
        dev = torch.device("cuda", 0)
        ec = inputs.ep_combine_inputs(world, 300, 4, 4, 16, 512, seed=19)
        experts = symmetric.SymmetricBuffer(256 + ec.max_rows * 512 * 2, device=dev)
        maps = symmetric.SymmetricBuffer(300 * 4 * 4, device=dev)
        experts.view(torch.bfloat16, (ec.max_rows, 512), 256).copy_(ec.expert_outputs[rank].to(dev))
        maps.view(torch.int32, (300, 4)).copy_(ec.inverse_maps[rank].to(dev))
        out = torch.empty(ec.counts[rank], 512, dtype=torch.bfloat16, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        symmetric.unpermute_reduce_scatter(out, experts, maps, torch.bfloat16, ec.max_rows, 512, 4,
                                           300, ec.rank_token_offset.to(dev),
                                           torch.tensor([300], dtype=torch.int32, device=dev),
                                           eo_byte_offset=256, dev_err=err)
        res = (rank, bits(out.cpu()), int(err))
        experts.close()
        maps.close()
        q.put(res)
    finally:
        dist.destroy_process_group()


def test_ep_combine_two_processes_cuda_ipc(cuda_device):
    """Two processes on this GPU, each publishing its expert rows and inverse
    map in CUDA-IPC-mapped buffers; the collective wrapper combines over both
    (host barriers under gloo; the kernels never wait on one another)."""
    import torch.multiprocessing as mp
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
    ec = inputs.ep_combine_inputs(world, 300, 4, 4, 16, 512, seed=19)
    for rank, got, err in res:
        assert err == 0
        want, _ = oracle.unpermute_reduce_scatter(
            [bits(e) for e in ec.expert_outputs], oracle.BF16, [bits(i) for i in ec.inverse_maps],
            300, rank, ec.rank_token_offset.numpy(), oracle.BF16,
            np.zeros((ec.counts[rank], 512), np.uint16), oracle.BF16)
        assert_bits_equal(got, want, f"rank {rank} over IPC")
