"""Tensor-level front end: shape checks, output allocation with torch, then the
C ABI (``_abi``).  torch is used for device memory and streams only; every
element of every output is produced by a kernel of libmoe_epilogue.so.
"""
from __future__ import annotations

import torch

from . import _abi
from ._abi import (MOE_ACT_SQRELU, MOE_ACT_SQRELU_CLAMP, MOE_ACT_SWIGLU,  # noqa: F401
                   MOE_BF16, MOE_FP16, MOE_FP32)

_DT = {torch.bfloat16: MOE_BF16, torch.float16: MOE_FP16, torch.float32: MOE_FP32}


def moe_dtype(dtype: torch.dtype) -> int:
    try:
        return _DT[dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {dtype}") from None


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")


def _rows_stride(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return t.stride(0)


def _flat_probs(probs: torch.Tensor, rows: int) -> torch.Tensor:
    if probs.dtype != torch.float32 or probs.numel() != rows or not probs.is_contiguous():
        raise ValueError("probs must be a contiguous fp32 tensor with one value per row")
    return probs


def swiglu_clamped_fwd(x, probs, limit, out=None, stream=None):
    """y = silu(clamp(gate, max=L)) * clamp(up, -L, L) * probs (bf16)."""
    _cuda(x, probs)
    rows, two_i = x.shape
    inter = two_i // 2
    if out is None:
        out = torch.empty(rows, inter, dtype=x.dtype, device=x.device)
    _abi.moe_swiglu_clamped_fwd(x, _flat_probs(probs, rows), out, rows, inter, _rows_stride(x),
                                _rows_stride(out), limit, moe_dtype(x.dtype), stream)
    return out


def swiglu_clamped_bwd(x, probs, grad_y, limit, grad_x=None, grad_probs=None, stream=None):
    """Returns (grad_x [rows, 2*inter] bf16, grad_probs [rows, 1] fp32)."""
    _cuda(x, probs, grad_y)
    rows, two_i = x.shape
    inter = two_i // 2
    if grad_x is None:
        grad_x = torch.empty_like(x)
    if grad_probs is None:
        grad_probs = torch.empty(rows, 1, dtype=torch.float32, device=x.device)
    _abi.moe_swiglu_clamped_bwd(x, _flat_probs(probs, rows), grad_y, grad_x, grad_probs, rows,
                                inter, _rows_stride(x), _rows_stride(grad_y),
                                _rows_stride(grad_x), limit, moe_dtype(x.dtype), stream)
    return grad_x, grad_probs


def _row_probs(probs: torch.Tensor, rows: int) -> torch.Tensor:
    if probs.numel() != rows or not probs.is_contiguous():
        raise ValueError("probs must be contiguous with one value per row")
    return probs


def router_weight_mul_fwd(x, probs, out_dtype=None, out=None, stream=None):
    """out = (x.float() * probs.float()).to(out_dtype); probs bf16, fp16 or fp32."""
    _cuda(x, probs)
    rows, hidden = x.shape
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    out_dtype = out_dtype or x.dtype
    if out is None:
        out = torch.empty(rows, hidden, dtype=out_dtype, device=x.device)
    _abi.moe_router_weight_mul_fwd_ex(x, moe_dtype(x.dtype), _row_probs(probs, rows),
                                      moe_dtype(probs.dtype), out, moe_dtype(out.dtype), rows,
                                      hidden, stream)
    return out


def router_weight_mul_bwd(grad_out, x, probs, x_dtype=None, grad_x=None, grad_probs=None,
                          stream=None):
    """Returns (grad_x, grad_probs or None); grad_probs has probs' dtype.  Pass
    x=None when the forward did not save x: then only grad_x is computed."""
    _cuda(grad_out, x, probs)
    rows, hidden = grad_out.shape
    x_dtype = x.dtype if x is not None else (x_dtype or grad_out.dtype)
    if grad_x is None:
        grad_x = torch.empty(rows, hidden, dtype=x_dtype, device=grad_out.device)
    if x is not None and grad_probs is None:
        grad_probs = torch.empty(rows, 1, dtype=probs.dtype, device=grad_out.device)
    _abi.moe_router_weight_mul_bwd_ex(grad_out, moe_dtype(grad_out.dtype), x, moe_dtype(x_dtype),
                                      _row_probs(probs, rows), moe_dtype(probs.dtype), grad_x,
                                      grad_probs if x is not None else None, rows, hidden, stream)
    return grad_x, (grad_probs if x is not None else None)


def act_with_probs_permuted(act, x, permutation_map, n_used, probs, clamp_scale=1.0,
                            zero_padding=False, out=None, dev_err=None, stream=None):
    """Activation with router probabilities over the padded, expert-grouped
    layout; act is MOE_ACT_SQRELU, MOE_ACT_SQRELU_CLAMP or MOE_ACT_SWIGLU."""
    _cuda(x, permutation_map, n_used, probs, dev_err)
    max_rows, cols = x.shape
    width = cols // 2 if act == MOE_ACT_SWIGLU else cols
    if out is None:
        out = torch.empty(max_rows, width, dtype=x.dtype, device=x.device)
    _abi.moe_act_with_probs_permuted(act, x, out, permutation_map, n_used, probs, probs.numel(),
                                     max_rows, width, clamp_scale, zero_padding, dev_err, stream)
    return out


def unpermute_ordered(expert_output, inverse_map, valid_tokens, out, dev_err=None, stream=None):
    """out[t] = sum over increasing local expert e of expert_output[inverse_map[t, e]]."""
    _cuda(expert_output, inverse_map, valid_tokens, out, dev_err)
    max_rows, hidden = expert_output.shape
    tokens, n_exp = inverse_map.shape
    _abi.moe_unpermute_ordered(expert_output, moe_dtype(expert_output.dtype), max_rows,
                               inverse_map, valid_tokens, out, moe_dtype(out.dtype), tokens,
                               hidden, n_exp, dev_err, stream)
    return out


def residual_add(expert_output, shared_expert_output, residual, out=None, stream=None):
    """out = residual + (expert_output + shared_expert_output), two roundings."""
    _cuda(expert_output, shared_expert_output, residual)
    if out is None:
        out = torch.empty_like(residual)
    _abi.moe_residual_add(expert_output, shared_expert_output, residual, out, residual.numel(),
                          moe_dtype(residual.dtype), stream)
    return out


def weighted_silu_mul_bounded(y, weights, bound_elems, num_programs=0, out=None, dev_err=None,
                              stream=None):
    """out[r, j] = bf16(silu(gate) * up * weights[r]) for flat elements below the
    device-resident bound_elems (int64); y is [rows, 2*half_n] (gate | up)."""
    _cuda(y, weights, bound_elems, dev_err)
    rows, two_h = y.shape
    half_n = two_h // 2
    if bound_elems.dtype != torch.int64:
        raise TypeError("bound_elems must be an int64 device tensor")
    if out is None:
        out = torch.empty(rows, half_n, dtype=y.dtype, device=y.device)
    _abi.moe_weighted_silu_mul_bounded(y, _flat_probs(weights, rows), out, bound_elems, rows,
                                       half_n, num_programs, dev_err, stream)
    return out


def epilogue_fused(expert_output, row_probs, inverse_map, valid_tokens, shared_expert_output,
                   residual, out=None, dev_err=None, stream=None):
    """residual + (unpermute(expert_output * row_probs) + shared), every rounding of
    the three-step chain kept, in one kernel."""
    _cuda(expert_output, row_probs, inverse_map, valid_tokens, shared_expert_output, residual,
          dev_err)
    max_rows, hidden = expert_output.shape
    tokens, n_exp = inverse_map.shape
    if out is None:
        out = torch.empty_like(residual)
    _abi.moe_epilogue_fused(expert_output, row_probs, max_rows, inverse_map, valid_tokens,
                            shared_expert_output, residual, out, tokens, hidden, n_exp,
                            moe_dtype(residual.dtype), dev_err, stream)
    return out


def pointer_table(tensors, device=None) -> torch.Tensor:
    """int64 [len(tensors)] device array of the tensors' data pointers, in order
    (the `buffers` argument of ordered_reduce_scatter_v for buffers that this
    GPU holds itself)."""
    device = device or tensors[0].device
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def ordered_reduce_scatter_v(buffers, rank, rank_token_offset, ep_tokens, capacity_rows, hidden,
                             in_dtype, local_tokens=None, out=None, out_dtype=None,
                             input_byte_offset=0, dev_err=None, stream=None):
    """This rank's rows of the rank-order fp32 reduce-scatter.

    buffers: int64 device tensor [world] of pointers (rank order) to each rank's
    [capacity_rows, hidden] block of `in_dtype` at `input_byte_offset`;
    rank_token_offset int32 [world] and ep_tokens int32 [1] on the device.
    Returns out [local_tokens, hidden] (`out_dtype`, default in_dtype).  The
    caller orders the launch against the other ranks' writes."""
    _cuda(buffers, rank_token_offset, ep_tokens, out, dev_err)
    if buffers.dtype != torch.int64 or buffers.dim() != 1:
        raise ValueError("buffers must be an int64 vector of device pointers")
    world = buffers.numel()
    if out is None:
        if local_tokens is None:
            raise ValueError("give local_tokens or out")
        out = torch.empty(local_tokens, hidden, dtype=out_dtype or in_dtype,
                          device=buffers.device)
    elif not out.is_contiguous() or out.dim() != 2 or out.shape[1] != hidden:
        raise ValueError("out must be a contiguous [local_tokens, hidden] tensor")
    _abi.moe_ordered_reduce_scatter_v(buffers, int(input_byte_offset), world, int(rank),
                                      rank_token_offset, ep_tokens, int(capacity_rows), out,
                                      out.shape[0], hidden, moe_dtype(in_dtype),
                                      moe_dtype(out.dtype), dev_err, stream)
    return out
