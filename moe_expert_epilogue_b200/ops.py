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
    """Every given tensor on one CUDA device (checked after the shape checks,
    just before the library call)."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on different devices: {dev} and {t.device}")


def _check(t, name, dtype=None, shape=None, numel=None, contiguous=True):
    """Dtype, shape (or element count) and contiguity of one argument; the C ABI
    trusts the sizes it is given, so a mismatch must stop here."""
    if t is None:
        return
    if dtype is not None:
        allowed = dtype if isinstance(dtype, tuple) else (dtype,)
        if t.dtype not in allowed:
            raise TypeError(f"{name}: dtype {t.dtype}, expected {' or '.join(map(str, allowed))}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: {t.numel()} elements, expected {numel}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_FLOATS = (torch.bfloat16, torch.float16, torch.float32)


def _rows_stride(t: torch.Tensor, name="tensor") -> int:
    if t.dim() != 2 or t.stride(1) != 1 or (t.shape[0] > 1 and t.stride(0) < t.shape[1]):
        raise ValueError(f"{name}: expected a 2-D tensor with unit column stride and "
                         "non-overlapping rows")
    return t.stride(0)


def _flat_probs(probs: torch.Tensor, rows: int, name="probs") -> torch.Tensor:
    _check(probs, name, dtype=torch.float32, numel=rows)
    return probs


def _two_d(t, name):
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    return t.shape


def swiglu_clamped_fwd(x, probs, limit, out=None, dev_err=None, stream=None):
    """y = silu(clamp(gate, max=L)) * clamp(up, -L, L) * probs, in x's dtype.
    dev_err (int32 [1], optional) receives MOE_DEVERR_TIMEOUT if a barrier
    wait of the TMA-staged kernel gave up."""
    rows, two_i = _two_d(x, "x")
    if two_i % 2:
        raise ValueError("x must hold [gate | up]: an even number of columns")
    inter = two_i // 2
    _check(x, "x", dtype=_FLOATS, contiguous=False)
    if out is None:
        out = torch.empty(rows, inter, dtype=x.dtype, device=x.device)
    _check(out, "out", dtype=x.dtype, shape=(rows, inter), contiguous=False)
    ld_x, ld_y = _rows_stride(x, "x"), _rows_stride(out, "out")
    _flat_probs(probs, rows)
    _check(dev_err, "dev_err", dtype=torch.int32, numel=1)
    _cuda(x, probs, out, dev_err)
    _abi.moe_swiglu_clamped_fwd_ex(x, probs, out, rows, inter, ld_x, ld_y, limit,
                                   moe_dtype(x.dtype), dev_err, stream)
    return out


def swiglu_clamped_bwd(x, probs, grad_y, limit, grad_x=None, grad_probs=None, stream=None):
    """Returns (grad_x [rows, 2*inter] in x's dtype, grad_probs [rows, 1] fp32)."""
    rows, two_i = _two_d(x, "x")
    if two_i % 2:
        raise ValueError("x must hold [gate | up]: an even number of columns")
    inter = two_i // 2
    _check(x, "x", dtype=_FLOATS, contiguous=False)
    _check(grad_y, "grad_y", dtype=x.dtype, shape=(rows, inter), contiguous=False)
    if grad_x is None:
        grad_x = torch.empty_like(x, memory_format=torch.contiguous_format)
    if grad_probs is None:
        grad_probs = torch.empty(rows, 1, dtype=torch.float32, device=x.device)
    _check(grad_x, "grad_x", dtype=x.dtype, shape=(rows, two_i), contiguous=False)
    _check(grad_probs, "grad_probs", dtype=torch.float32, numel=rows)
    ld_x, ld_gy, ld_gx = (_rows_stride(x, "x"), _rows_stride(grad_y, "grad_y"),
                          _rows_stride(grad_x, "grad_x"))
    _flat_probs(probs, rows)
    _cuda(x, probs, grad_y, grad_x, grad_probs)
    _abi.moe_swiglu_clamped_bwd(x, probs, grad_y, grad_x, grad_probs, rows, inter, ld_x, ld_gy,
                                ld_gx, limit, moe_dtype(x.dtype), stream)
    return grad_x, grad_probs


def router_weight_mul_fwd(x, probs, out_dtype=None, out=None, stream=None):
    """out = (x.float() * probs.float()).to(out_dtype); probs bf16, fp16 or fp32."""
    rows, hidden = _two_d(x, "x")
    _check(x, "x", dtype=_FLOATS)
    _check(probs, "probs", dtype=_FLOATS, numel=rows)
    if out is None:
        out = torch.empty(rows, hidden, dtype=out_dtype or x.dtype, device=x.device)
    _check(out, "out", dtype=_FLOATS, shape=(rows, hidden))
    _cuda(x, probs, out)
    _abi.moe_router_weight_mul_fwd_ex(x, moe_dtype(x.dtype), probs, moe_dtype(probs.dtype), out,
                                      moe_dtype(out.dtype), rows, hidden, stream)
    return out


def router_weight_mul_bwd(grad_out, x, probs, x_dtype=None, grad_x=None, grad_probs=None,
                          stream=None):
    """Returns (grad_x, grad_probs or None); grad_probs has probs' dtype.  Pass
    x=None when the forward did not save x: then only grad_x is computed."""
    rows, hidden = _two_d(grad_out, "grad_out")
    _check(grad_out, "grad_out", dtype=_FLOATS)
    _check(x, "x", dtype=_FLOATS, shape=(rows, hidden))
    _check(probs, "probs", dtype=_FLOATS, numel=rows)
    x_dtype = x.dtype if x is not None else (x_dtype or grad_out.dtype)
    if grad_x is None:
        grad_x = torch.empty(rows, hidden, dtype=x_dtype, device=grad_out.device)
    _check(grad_x, "grad_x", dtype=x_dtype, shape=(rows, hidden))
    if x is None:
        grad_probs = None
    elif grad_probs is None:
        grad_probs = torch.empty(rows, 1, dtype=probs.dtype, device=grad_out.device)
    _check(grad_probs, "grad_probs", dtype=probs.dtype, numel=rows)
    _cuda(grad_out, x, probs, grad_x, grad_probs)
    _abi.moe_router_weight_mul_bwd_ex(grad_out, moe_dtype(grad_out.dtype), x, moe_dtype(x_dtype),
                                      probs, moe_dtype(probs.dtype), grad_x, grad_probs, rows,
                                      hidden, stream)
    return grad_x, grad_probs


def act_with_probs_permuted(act, x, permutation_map, n_used, probs, clamp_scale=1.0,
                            zero_padding=False, out=None, dev_err=None, stream=None):
    """Activation with router probabilities over the padded, expert-grouped
    layout (bf16); act is MOE_ACT_SQRELU, MOE_ACT_SQRELU_CLAMP or MOE_ACT_SWIGLU."""
    max_rows, cols = _two_d(x, "x")
    if act == MOE_ACT_SWIGLU and cols % 2:
        raise ValueError("SwiGLU input must hold [gate | up]: an even number of columns")
    width = cols // 2 if act == MOE_ACT_SWIGLU else cols
    _check(x, "x", dtype=torch.bfloat16)
    _check(permutation_map, "permutation_map", dtype=torch.int32, numel=max_rows)
    _check(n_used, "n_used", dtype=torch.int32, numel=1)
    _check(probs, "probs", dtype=torch.float32)
    _check(dev_err, "dev_err", dtype=torch.int32, numel=1)
    if out is None:
        out = torch.empty(max_rows, width, dtype=x.dtype, device=x.device)
    _check(out, "out", dtype=torch.bfloat16, shape=(max_rows, width))
    _cuda(x, permutation_map, n_used, probs, out, dev_err)
    _abi.moe_act_with_probs_permuted(act, x, out, permutation_map, n_used, probs, probs.numel(),
                                     max_rows, width, clamp_scale, zero_padding, dev_err, stream)
    return out


def unpermute_ordered(expert_output, inverse_map, valid_tokens, out, dev_err=None, stream=None):
    """out[t] = sum over increasing local expert e of expert_output[inverse_map[t, e]]."""
    max_rows, hidden = _two_d(expert_output, "expert_output")
    tokens, n_exp = _two_d(inverse_map, "inverse_map")
    _check(expert_output, "expert_output", dtype=_FLOATS)
    _check(inverse_map, "inverse_map", dtype=torch.int32)
    _check(valid_tokens, "valid_tokens", dtype=torch.int32, numel=1)
    _check(out, "out", dtype=_FLOATS, shape=(tokens, hidden))
    _check(dev_err, "dev_err", dtype=torch.int32, numel=1)
    _cuda(expert_output, inverse_map, valid_tokens, out, dev_err)
    _abi.moe_unpermute_ordered(expert_output, moe_dtype(expert_output.dtype), max_rows,
                               inverse_map, valid_tokens, out, moe_dtype(out.dtype), tokens,
                               hidden, n_exp, dev_err, stream)
    return out


def residual_add(expert_output, shared_expert_output, residual, out=None, stream=None):
    """out = residual + (expert_output + shared_expert_output), two roundings;
    out may be residual itself (in place)."""
    _check(residual, "residual", dtype=_FLOATS)
    for t, name in ((expert_output, "expert_output"),
                    (shared_expert_output, "shared_expert_output")):
        _check(t, name, dtype=residual.dtype, shape=residual.shape)
    if out is None:
        out = torch.empty_like(residual)
    _check(out, "out", dtype=residual.dtype, shape=residual.shape)
    _cuda(expert_output, shared_expert_output, residual, out)
    _abi.moe_residual_add(expert_output, shared_expert_output, residual, out, residual.numel(),
                          moe_dtype(residual.dtype), stream)
    return out


def weighted_silu_mul_bounded(y, weights, bound_elems, num_programs=0, out=None, dev_err=None,
                              stream=None):
    """out[r, j] = bf16(silu(gate) * up * weights[r]) for flat elements below the
    device-resident bound_elems (int64); y is [rows, 2*half_n] (gate | up)."""
    rows, two_h = _two_d(y, "y")
    if two_h % 2:
        raise ValueError("y must hold [gate | up]: an even number of columns")
    half_n = two_h // 2
    _check(y, "y", dtype=torch.bfloat16)
    _check(bound_elems, "bound_elems", dtype=torch.int64, numel=1)
    _check(dev_err, "dev_err", dtype=torch.int32, numel=1)
    _flat_probs(weights, rows, "weights")
    if out is None:
        out = torch.empty(rows, half_n, dtype=y.dtype, device=y.device)
    _check(out, "out", dtype=torch.bfloat16, shape=(rows, half_n))
    _cuda(y, weights, bound_elems, out, dev_err)
    _abi.moe_weighted_silu_mul_bounded(y, weights, out, bound_elems, rows, half_n, num_programs,
                                       dev_err, stream)
    return out


def epilogue_fused(expert_output, row_probs, inverse_map, valid_tokens, shared_expert_output,
                   residual, out=None, dev_err=None, stream=None):
    """residual + (unpermute(expert_output * row_probs) + shared), every rounding of
    the three-step chain kept, in one kernel; out may be residual (in place)."""
    max_rows, hidden = _two_d(expert_output, "expert_output")
    tokens, n_exp = _two_d(inverse_map, "inverse_map")
    _check(residual, "residual", dtype=_FLOATS, shape=(tokens, hidden))
    dt = residual.dtype
    _check(expert_output, "expert_output", dtype=dt)
    _check(shared_expert_output, "shared_expert_output", dtype=dt, shape=(tokens, hidden))
    _flat_probs(row_probs, max_rows, "row_probs")
    _check(inverse_map, "inverse_map", dtype=torch.int32)
    _check(valid_tokens, "valid_tokens", dtype=torch.int32, numel=1)
    _check(dev_err, "dev_err", dtype=torch.int32, numel=1)
    if out is None:
        out = torch.empty_like(residual)
    _check(out, "out", dtype=dt, shape=(tokens, hidden))
    _cuda(expert_output, row_probs, inverse_map, valid_tokens, shared_expert_output, residual,
          out, dev_err)
    _abi.moe_epilogue_fused(expert_output, row_probs, max_rows, inverse_map, valid_tokens,
                            shared_expert_output, residual, out, tokens, hidden, n_exp,
                            moe_dtype(dt), dev_err, stream)
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
    if buffers.dim() != 1:
        raise ValueError("buffers must be a vector of device pointers")
    _check(buffers, "buffers", dtype=torch.int64)
    world = buffers.numel()
    _check(rank_token_offset, "rank_token_offset", dtype=torch.int32, numel=world)
    _check(ep_tokens, "ep_tokens", dtype=torch.int32, numel=1)
    _check(dev_err, "dev_err", dtype=torch.int32, numel=1)
    if out is None:
        if local_tokens is None:
            raise ValueError("give local_tokens or out")
        out = torch.empty(local_tokens, hidden, dtype=out_dtype or in_dtype,
                          device=buffers.device)
    _two_d(out, "out")
    _check(out, "out", dtype=_FLOATS, shape=(out.shape[0], hidden))
    _cuda(buffers, rank_token_offset, ep_tokens, out, dev_err)
    _abi.moe_ordered_reduce_scatter_v(buffers, int(input_byte_offset), world, int(rank),
                                      rank_token_offset, ep_tokens, int(capacity_rows), out,
                                      out.shape[0], hidden, moe_dtype(in_dtype),
                                      moe_dtype(out.dtype), dev_err, stream)
    return out


def unpermute_reduce_scatter(expert_outputs, eo_dtype, max_rows, inverse_maps, num_local_experts,
                             capacity_rows, ep_tokens, rank, rank_token_offset, hidden,
                             local_tokens=None, out=None, out_dtype=None, partial_dtype=None,
                             dev_err=None, stream=None):
    """This rank's rows of the EP combine: every rank's fixed-order unpermute
    and the rank-order reduce-scatter of the results, in one kernel.

    expert_outputs, inverse_maps: int64 device tensors [world] of pointers
    (rank order) to each rank's [max_rows, hidden] expert rows of `eo_dtype`
    and int32 [capacity_rows, num_local_experts] inverse map; ep_tokens int32
    [1] and rank_token_offset int32 [world] on the device.  partial_dtype
    (default eo_dtype) is the dtype the two-step form would store its partial
    sums in.  Returns out [local_tokens, hidden] (out_dtype, default eo_dtype)."""
    for t, name in ((expert_outputs, "expert_outputs"), (inverse_maps, "inverse_maps")):
        if t.dim() != 1:
            raise ValueError(f"{name} must be a vector of device pointers")
        _check(t, name, dtype=torch.int64)
    world = expert_outputs.numel()
    _check(inverse_maps, "inverse_maps", numel=world)
    _check(rank_token_offset, "rank_token_offset", dtype=torch.int32, numel=world)
    _check(ep_tokens, "ep_tokens", dtype=torch.int32, numel=1)
    _check(dev_err, "dev_err", dtype=torch.int32, numel=1)
    if out is None:
        if local_tokens is None:
            raise ValueError("give local_tokens or out")
        out = torch.empty(local_tokens, hidden, dtype=out_dtype or eo_dtype,
                          device=expert_outputs.device)
    _two_d(out, "out")
    _check(out, "out", dtype=_FLOATS, shape=(out.shape[0], hidden))
    _cuda(expert_outputs, inverse_maps, rank_token_offset, ep_tokens, out, dev_err)
    _abi.moe_unpermute_reduce_scatter(expert_outputs, moe_dtype(eo_dtype), int(max_rows),
                                      inverse_maps, int(num_local_experts), int(capacity_rows),
                                      ep_tokens, world, int(rank), rank_token_offset,
                                      moe_dtype(partial_dtype or eo_dtype), out,
                                      moe_dtype(out.dtype), out.shape[0], hidden, dev_err, stream)
    return out
