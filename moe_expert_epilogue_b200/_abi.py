"""ctypes binding of the C ABI declared in include/moe_epilogue.h.

Argument marshalling only: every function here has the name and the argument
order of its C counterpart, turns tensors into device pointers and a stream
into its handle, calls the library and raises :class:`MoeError` on a non-OK
status.  All arithmetic happens in the CUDA kernels of libmoe_epilogue.so;
there is no Python or CPU fallback -- if the library is missing, the first
call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_epilogue.so")

MOE_BF16, MOE_FP16, MOE_FP32 = 0, 1, 2
MOE_ACT_SQRELU, MOE_ACT_SQRELU_CLAMP, MOE_ACT_SWIGLU = 0, 1, 2
(MOE_OK, MOE_ERR_NULL, MOE_ERR_SHAPE, MOE_ERR_DTYPE, MOE_ERR_ALIGN, MOE_ERR_LIMIT,
 MOE_ERR_CUDA) = range(7)
MOE_DEVERR_COUNT, MOE_DEVERR_MAP, MOE_DEVERR_INVERSE, MOE_DEVERR_TIMEOUT = 1, 2, 4, 8

_P, _I64, _I32, _F, _I = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                          ctypes.c_int)

# name -> argtypes (every entry point returns int)
SIGNATURES = {
    "moe_swiglu_clamped_fwd": [_P, _P, _P, _I64, _I64, _I64, _I64, _F, _I, _P],
    "moe_swiglu_clamped_fwd_ex": [_P, _P, _P, _I64, _I64, _I64, _I64, _F, _I, _P, _P],
    "moe_test_swiglu_fwd_stalled": [_P, _P, _P, _I64, _I64, _F, _I, _I32, _I64, _I64, _P, _P],
    "moe_swiglu_clamped_bwd": [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _F, _I, _P],
    "moe_router_weight_mul_fwd": [_P, _I, _P, _P, _I, _I64, _I64, _P],
    "moe_router_weight_mul_bwd": [_P, _I, _P, _I, _P, _P, _P, _I64, _I64, _P],
    "moe_router_weight_mul_fwd_ex": [_P, _I, _P, _I, _P, _I, _I64, _I64, _P],
    "moe_router_weight_mul_bwd_ex": [_P, _I, _P, _I, _P, _I, _P, _P, _I64, _I64, _P],
    "moe_act_with_probs_permuted": [_I, _P, _P, _P, _P, _P, _I64, _I64, _I64, _F, _I, _P, _P],
    "moe_unpermute_ordered": [_P, _I, _I64, _P, _P, _P, _I, _I64, _I64, _I32, _P, _P],
    "moe_residual_add": [_P, _P, _P, _P, _I64, _I, _P],
    "moe_weighted_silu_mul_bounded": [_P, _P, _P, _P, _I64, _I64, _I32, _P, _P],
    "moe_epilogue_fused": [_P, _P, _I64, _P, _P, _P, _P, _P, _I64, _I64, _I32, _I, _P, _P],
    "moe_ordered_reduce_scatter_v": [_P, _I64, _I32, _I32, _P, _P, _I64, _P, _I64, _I64, _I, _I,
                                     _P, _P],
    "moe_unpermute_reduce_scatter": [_P, _I, _I64, _P, _I32, _I64, _P, _I32, _I32, _P, _I, _P,
                                     _I, _I64, _I64, _P, _P],
    "moe_symm_alloc": [ctypes.c_size_t, ctypes.POINTER(_P)],
    "moe_symm_free": [_P],
    "moe_ipc_export": [_P, ctypes.c_char_p],
    "moe_ipc_open": [ctypes.c_char_p, ctypes.POINTER(_P)],
    "moe_ipc_close": [_P],
}

MOE_IPC_HANDLE_BYTES = 64

_lock = threading.Lock()
_lib = None


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib().moe_status_string(status).decode()
        if status == MOE_ERR_CUDA:
            msg += f" (cudaError {lib().moe_last_cuda_error()})"
        super().__init__(f"{fn}: {msg}")


def lib() -> ctypes.CDLL:
    """Load libmoe_epilogue.so (built in-tree); raise if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m moe_expert_epilogue_b200.build` (needs nvcc)")
            L = ctypes.CDLL(LIB_PATH)
            L.moe_status_string.restype = ctypes.c_char_p
            L.moe_status_string.argtypes = [_I]
            L.moe_last_cuda_error.restype = _I
            L.moe_last_cuda_error.argtypes = []
            L.moe_abi_version.restype = _I
            L.moe_abi_version.argtypes = []
            L.moe_device_errors.restype = _I
            L.moe_device_errors.argtypes = [ctypes.POINTER(_I32), _I]
            for name, args in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = _I
                fn.argtypes = args
            _lib = L
    return _lib


def ptr(a) -> int | None:
    """A device pointer from a tensor (its data_ptr), an int, or None."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def stream_handle(stream) -> int | None:
    """cudaStream_t from None (torch's current stream), a torch stream or an int."""
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _call(name, *args):
    rc = getattr(lib(), name)(*args)
    if rc != MOE_OK:
        raise MoeError(name, rc)


def moe_swiglu_clamped_fwd(x, probs, y, rows, inter, ld_x, ld_y, limit, dt=MOE_BF16,
                           stream=None):
    _call("moe_swiglu_clamped_fwd", ptr(x), ptr(probs), ptr(y), rows, inter, ld_x, ld_y,
          float(limit), dt, stream_handle(stream))


def moe_swiglu_clamped_fwd_ex(x, probs, y, rows, inter, ld_x, ld_y, limit, dt=MOE_BF16,
                              dev_err=None, stream=None):
    _call("moe_swiglu_clamped_fwd_ex", ptr(x), ptr(probs), ptr(y), rows, inter, ld_x, ld_y,
          float(limit), dt, ptr(dev_err), stream_handle(stream))


def moe_test_swiglu_fwd_stalled(x, probs, y, rows, inter, limit, dt, grid, stall_row,
                                wait_cycles, dev_err, stream=None):
    _call("moe_test_swiglu_fwd_stalled", ptr(x), ptr(probs), ptr(y), rows, inter, float(limit),
          dt, grid, stall_row, wait_cycles, ptr(dev_err), stream_handle(stream))


def moe_swiglu_clamped_bwd(x, probs, grad_y, grad_x, grad_probs, rows, inter, ld_x, ld_gy,
                           ld_gx, limit, dt=MOE_BF16, stream=None):
    _call("moe_swiglu_clamped_bwd", ptr(x), ptr(probs), ptr(grad_y), ptr(grad_x),
          ptr(grad_probs), rows, inter, ld_x, ld_gy, ld_gx, float(limit), dt,
          stream_handle(stream))


def moe_router_weight_mul_fwd(x, x_dt, probs, out, out_dt, rows, hidden, stream=None):
    _call("moe_router_weight_mul_fwd", ptr(x), x_dt, ptr(probs), ptr(out), out_dt, rows, hidden,
          stream_handle(stream))


def moe_router_weight_mul_bwd(grad_out, g_dt, x, x_dt, probs, grad_x, grad_probs, rows, hidden,
                              stream=None):
    _call("moe_router_weight_mul_bwd", ptr(grad_out), g_dt, ptr(x), x_dt, ptr(probs),
          ptr(grad_x), ptr(grad_probs), rows, hidden, stream_handle(stream))


def moe_router_weight_mul_fwd_ex(x, x_dt, probs, probs_dt, out, out_dt, rows, hidden,
                                 stream=None):
    _call("moe_router_weight_mul_fwd_ex", ptr(x), x_dt, ptr(probs), probs_dt, ptr(out), out_dt,
          rows, hidden, stream_handle(stream))


def moe_router_weight_mul_bwd_ex(grad_out, g_dt, x, x_dt, probs, probs_dt, grad_x, grad_probs,
                                 rows, hidden, stream=None):
    _call("moe_router_weight_mul_bwd_ex", ptr(grad_out), g_dt, ptr(x), x_dt, ptr(probs), probs_dt,
          ptr(grad_x), ptr(grad_probs), rows, hidden, stream_handle(stream))


def moe_act_with_probs_permuted(act, x, out, permutation_map, n_used, probs, num_probs,
                                max_rows, width, clamp_scale, zero_padding, dev_err=None,
                                stream=None):
    _call("moe_act_with_probs_permuted", act, ptr(x), ptr(out), ptr(permutation_map),
          ptr(n_used), ptr(probs), num_probs, max_rows, width, float(clamp_scale),
          int(bool(zero_padding)), ptr(dev_err), stream_handle(stream))


def moe_unpermute_ordered(expert_output, in_dt, max_rows, inverse_map, valid_tokens, out,
                          out_dt, tokens, hidden, num_local_experts, dev_err=None,
                          stream=None):
    _call("moe_unpermute_ordered", ptr(expert_output), in_dt, max_rows, ptr(inverse_map),
          ptr(valid_tokens), ptr(out), out_dt, tokens, hidden, num_local_experts, ptr(dev_err),
          stream_handle(stream))


def moe_residual_add(expert_output, shared_expert_output, residual, out, numel, dt,
                     stream=None):
    _call("moe_residual_add", ptr(expert_output), ptr(shared_expert_output), ptr(residual),
          ptr(out), numel, dt, stream_handle(stream))


def moe_weighted_silu_mul_bounded(y, weights, out, bound_elems, rows, half_n, num_programs=0,
                                  dev_err=None, stream=None):
    _call("moe_weighted_silu_mul_bounded", ptr(y), ptr(weights), ptr(out), ptr(bound_elems), rows,
          half_n, num_programs, ptr(dev_err), stream_handle(stream))


def moe_epilogue_fused(expert_output, row_probs, max_rows, inverse_map, valid_tokens,
                       shared_expert_output, residual, out, tokens, hidden, num_local_experts,
                       dt, dev_err=None, stream=None):
    _call("moe_epilogue_fused", ptr(expert_output), ptr(row_probs), max_rows, ptr(inverse_map),
          ptr(valid_tokens), ptr(shared_expert_output), ptr(residual), ptr(out), tokens, hidden,
          num_local_experts, dt, ptr(dev_err), stream_handle(stream))


def moe_ordered_reduce_scatter_v(buffers, input_byte_offset, world, rank, rank_token_offset,
                                 ep_tokens, capacity_rows, out, local_tokens, hidden, in_dt,
                                 out_dt, dev_err=None, stream=None):
    _call("moe_ordered_reduce_scatter_v", ptr(buffers), input_byte_offset, world, rank,
          ptr(rank_token_offset), ptr(ep_tokens), capacity_rows, ptr(out), local_tokens, hidden,
          in_dt, out_dt, ptr(dev_err), stream_handle(stream))


def moe_unpermute_reduce_scatter(expert_outputs, eo_dt, max_rows, inverse_maps,
                                 num_local_experts, capacity_rows, ep_tokens, world, rank,
                                 rank_token_offset, partial_dt, out, out_dt, local_tokens, hidden,
                                 dev_err=None, stream=None):
    _call("moe_unpermute_reduce_scatter", ptr(expert_outputs), eo_dt, max_rows, ptr(inverse_maps),
          num_local_experts, capacity_rows, ptr(ep_tokens), world, rank, ptr(rank_token_offset),
          partial_dt, ptr(out), out_dt, local_tokens, hidden, ptr(dev_err), stream_handle(stream))


def moe_symm_alloc(nbytes: int) -> int:
    """A zero-filled device allocation of `nbytes` on the current device."""
    p = _P(0)
    _call("moe_symm_alloc", nbytes, ctypes.byref(p))
    return int(p.value)


def moe_symm_free(p: int) -> None:
    _call("moe_symm_free", p)


def moe_ipc_export(p: int) -> bytes:
    """The MOE_IPC_HANDLE_BYTES-byte IPC handle of an moe_symm_alloc allocation."""
    buf = ctypes.create_string_buffer(MOE_IPC_HANDLE_BYTES)
    _call("moe_ipc_export", p, buf)
    return buf.raw


def moe_ipc_open(handle: bytes) -> int:
    """Maps another process's allocation into this one; returns its pointer."""
    if len(handle) != MOE_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle has MOE_IPC_HANDLE_BYTES bytes")
    p = _P(0)
    _call("moe_ipc_open", handle, ctypes.byref(p))
    return int(p.value)


def moe_ipc_close(p: int) -> None:
    _call("moe_ipc_close", p)


def moe_device_errors(clear=True) -> int:
    """Error bits recorded on the current device by kernels without a dev_err
    argument (MOE_DEVERR_TIMEOUT); synchronous."""
    v = _I32(0)
    _call("moe_device_errors", ctypes.byref(v), int(bool(clear)))
    return int(v.value)
