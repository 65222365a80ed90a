"""Rank-order reduce-scatter and EP combine between the processes of one node.

(core.inference.moe.batch_invariant: ordered_reduce_scatter_v.)  Every EP rank
writes its partial results for the tokens of all ranks into a buffer that every
other rank can read (`SymmetricBuffer`); `ordered_reduce_scatter_v` then sums,
on each rank, the rows that rank owns over all ranks in rank order (fp32, one
rounding), reading the peers' buffers directly over NVLink with plain loads;
`unpermute_reduce_scatter` does the same straight from every rank's expert
rows (the unpermute fused in).

Ordering is stream-ordered and host-free: a one-element all-reduce on the
process group before the launch (every rank's inputs are complete) and after
it (no rank reuses its buffer while a peer still reads it) -- the job the
pages give to the symmetric-memory signal pads.  The kernel itself waits on
nothing, so a missing rank surfaces as the process group's timeout on the
host, never as a spinning GPU.

The buffers are plain device allocations mapped into every process with CUDA
IPC (`moe_symm_alloc`, `moe_ipc_export`, `moe_ipc_open` in the C ABI); the
mapping backend is a parameter so that the exchange protocol can be exercised
on CPU with a stand-in.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _abi, ops


class _DeviceBytes:
    """A raw device range seen by torch through the CUDA array interface."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1",
                                         "data": (ptr, False), "strides": None,
                                         "version": 2}


class CudaIpc:
    """Mapping backend of the C ABI: device allocations shared with CUDA IPC."""

    alloc = staticmethod(_abi.moe_symm_alloc)
    free = staticmethod(_abi.moe_symm_free)
    export = staticmethod(_abi.moe_ipc_export)
    open = staticmethod(_abi.moe_ipc_open)
    close = staticmethod(_abi.moe_ipc_close)

    @staticmethod
    def view(ptr: int, nbytes: int, device) -> torch.Tensor:
        return torch.as_tensor(_DeviceBytes(ptr, nbytes), device=device)

    @staticmethod
    def table(ptrs, device) -> torch.Tensor:
        return torch.tensor(ptrs, dtype=torch.int64, device=device)


class SymmetricBuffer:
    """`nbytes` of device memory on every rank of `group`, every rank's buffer
    mapped into every process.  `ptrs[q]` is rank q's buffer as this process
    addresses it; `table` is the same list as a device int64 tensor (the
    `buffers` argument of the reduce-scatter).  Collective: every rank of the
    group constructs it together, and closes it together."""

    def __init__(self, nbytes: int, group=None, device=None, backend=None):
        self.group = group
        self.backend = backend or CudaIpc()
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.device = device if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        self.nbytes = int(nbytes)
        self.local = self.backend.alloc(self.nbytes)
        handles = [None] * self.world
        dist.all_gather_object(handles, self.backend.export(self.local), group=group)
        self.ptrs = []
        try:
            for q, h in enumerate(handles):
                self.ptrs.append(self.local if q == self.rank else self.backend.open(h))
        except Exception:
            self._release()
            raise
        self.table = self.backend.table(self.ptrs, self.device)
        self.closed = False

    def view(self, dtype: torch.dtype, shape, byte_offset: int = 0) -> torch.Tensor:
        """This rank's buffer from `byte_offset` as a tensor (valid until close())."""
        numel = 1
        for s in shape:
            numel *= int(s)
        esize = torch.empty((), dtype=dtype).element_size()
        if byte_offset < 0 or byte_offset % esize or byte_offset + numel * esize > self.nbytes:
            raise ValueError("view outside the buffer or misaligned")
        raw = self.backend.view(self.local, self.nbytes, self.device)
        return raw[byte_offset:byte_offset + numel * esize].view(dtype).view(*shape)

    def table_at(self, byte_offset: int = 0) -> torch.Tensor:
        """The ranks' buffers from `byte_offset`, as a device pointer table."""
        if byte_offset < 0 or byte_offset >= max(1, self.nbytes):
            raise ValueError("offset outside the buffer")
        return self.backend.table([p + byte_offset for p in self.ptrs], self.device)

    def _release(self):
        for q, p in enumerate(self.ptrs):
            if q != self.rank:
                self.backend.close(p)
        self.ptrs = []
        self.backend.free(self.local)

    def close(self):
        """Collective: waits until no rank can still read this buffer, then
        unmaps the peers and frees the local allocation."""
        if self.closed:
            return
        stream_barrier(self.group, self.device)
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        self._release()
        self.closed = True


def stream_barrier(group=None, device=None):
    """No rank's later work starts before every rank's earlier work is done: a
    one-element all-reduce on the group.  Under NCCL it is stream-ordered (the
    current stream waits on it; the host does not).  Under any other backend
    it is a host barrier, so a CUDA device is synchronised first."""
    is_cuda = device is not None and getattr(device, "type", "cpu") == "cuda"
    if is_cuda and dist.get_backend(group) == "nccl":
        flag = torch.zeros(1, dtype=torch.int32, device=device)
    else:
        if is_cuda:
            torch.cuda.synchronize(device)
        flag = torch.zeros(1, dtype=torch.int32)
    dist.all_reduce(flag, group=group)


def ordered_reduce_scatter_v(output: torch.Tensor, symm: SymmetricBuffer,
                             rank_token_offset: torch.Tensor, ep_tokens: torch.Tensor,
                             capacity_rows: int, hidden: int, in_dtype: torch.dtype,
                             input_byte_offset: int = 0, dev_err=None,
                             launch_hooks=None) -> torch.Tensor:
    """Collective over symm.group: this rank's `output` [local_tokens, hidden]
    = the rank-order fp32 sum of its token rows over every rank's block
    ([capacity_rows, hidden] of in_dtype at input_byte_offset in the symmetric
    buffer), launched on the current stream between two stream barriers.
    `launch_hooks`, a (before, after) pair of callables, runs just around the
    launch, inside the barriers (e.g. to record timing events)."""
    esize = torch.empty((), dtype=in_dtype).element_size()
    if input_byte_offset + capacity_rows * hidden * esize > symm.nbytes:
        raise ValueError("the input block does not fit in the symmetric buffer")
    stream_barrier(symm.group, symm.device)
    if launch_hooks:
        launch_hooks[0]()
    ops.ordered_reduce_scatter_v(symm.table, symm.rank, rank_token_offset, ep_tokens,
                                 capacity_rows, hidden, in_dtype, out=output,
                                 input_byte_offset=input_byte_offset, dev_err=dev_err)
    if launch_hooks:
        launch_hooks[1]()
    stream_barrier(symm.group, symm.device)
    return output


def unpermute_reduce_scatter(output: torch.Tensor, experts: SymmetricBuffer,
                             inverse_maps: SymmetricBuffer, eo_dtype: torch.dtype, max_rows: int,
                             hidden: int, num_local_experts: int, capacity_rows: int,
                             rank_token_offset: torch.Tensor, ep_tokens: torch.Tensor,
                             eo_byte_offset: int = 0, inv_byte_offset: int = 0,
                             partial_dtype=None, dev_err=None, launch_hooks=None) -> torch.Tensor:
    """Collective over experts.group: the EP combine.  Every rank holds its
    experts' output rows ([max_rows, hidden] of eo_dtype at eo_byte_offset of
    `experts`) and its inverse map over the token rows of all ranks (int32
    [capacity_rows, num_local_experts] at inv_byte_offset of `inverse_maps`);
    this rank's `output` [local_tokens, hidden] gets, per token, every rank's
    expert-order partial sum folded in rank order -- the unpermute and the
    rank-order reduce-scatter in one kernel, launched on the current stream
    between two stream barriers (`launch_hooks` as for ordered_reduce_scatter_v)."""
    esize = torch.empty((), dtype=eo_dtype).element_size()
    if eo_byte_offset + max_rows * hidden * esize > experts.nbytes or \
            inv_byte_offset + capacity_rows * num_local_experts * 4 > inverse_maps.nbytes:
        raise ValueError("a block does not fit in its symmetric buffer")
    if experts.world != inverse_maps.world or experts.rank != inverse_maps.rank:
        raise ValueError("both buffers must span the same group")
    stream_barrier(experts.group, experts.device)
    if launch_hooks:
        launch_hooks[0]()
    ops.unpermute_reduce_scatter(experts.table_at(eo_byte_offset), eo_dtype, max_rows,
                                 inverse_maps.table_at(inv_byte_offset), num_local_experts,
                                 capacity_rows, ep_tokens, experts.rank, rank_token_offset,
                                 hidden, out=output, partial_dtype=partial_dtype,
                                 dev_err=dev_err)
    if launch_hooks:
        launch_hooks[1]()
    stream_barrier(experts.group, experts.device)
    return output
