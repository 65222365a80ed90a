"""Plain CPU oracle for the MoE expert-epilogue ops (numpy front end).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``moe_expert_epilogue_b200``) never imports it, and the two share
no code: the arithmetic lives in ``moe_oracle.c`` (plain C, fp32 evaluation of
each documented formula, one rounding to the storage dtype), built here into
``libmoe_oracle.so`` with gcc and called through ctypes.

Array conventions: bf16 and fp16 tensors are passed as ``numpy.uint16`` arrays
holding the raw bits; fp32 as ``numpy.float32``; index maps as ``numpy.int32``.
Every function allocates and returns its outputs.

Pins: see ``tests/test_oracle_pins.py``.  Every op has at least one pin that is
independent of this code (library routines, closed forms, float64 finite
differences, brute force on tiny inputs); no function is left unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_LOCK = threading.Lock()
_LIB = None

BF16, F16, F32 = 0, 1, 2
SQRELU, SQRELU_CLAMP, SWIGLU = 0, 1, 2
ERR_COUNT, ERR_MAP, ERR_INVERSE = 1, 2, 4

_CFLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction, no fast math)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load(path: str) -> ctypes.CDLL:
    """Load an oracle build at `path` and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P, I64, I32, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    sig = {
        "orc_bf16_from_f32": (ctypes.c_uint16, [F]),
        "orc_f32_from_bf16": (F, [ctypes.c_uint16]),
        "orc_f16_from_f32": (ctypes.c_uint16, [F]),
        "orc_f32_from_f16": (F, [ctypes.c_uint16]),
        "orc_swiglu_clamped_fwd": (None, [P, P, P, I64, I64, I64, I64, F]),
        "orc_swiglu_clamped_bwd": (None, [P, P, P, P, P, P, I64, I64, I64, I64, I64, F]),
        "orc_swiglu_clamped_fwd_f64": (None, [P, P, P, P, I64, ctypes.c_double]),
        "orc_swiglu_clamped_fwd_dt": (None, [P, P, P, I64, I64, I64, I64, F, ctypes.c_int]),
        "orc_swiglu_clamped_bwd_dt": (None, [P, P, P, P, P, P, I64, I64, I64, I64, I64, F,
                                             ctypes.c_int]),
        "orc_router_weight_fwd": (None, [P, ctypes.c_int, P, P, ctypes.c_int, I64, I64]),
        "orc_router_weight_fwd_p": (None, [P, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int,
                                           I64, I64]),
        "orc_router_weight_bwd_p": (None, [P, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int, P,
                                           P, P, I64, I64]),
        "orc_router_weight_bwd": (None, [P, ctypes.c_int, P, ctypes.c_int, P, P, P, P,
                                         I64, I64]),
        "orc_act_with_probs_permuted": (ctypes.c_int, [ctypes.c_int, P, P, P, I32, P, I64,
                                                       I64, I64, F, ctypes.c_int]),
        "orc_unpermute_ordered": (ctypes.c_int, [P, ctypes.c_int, I64, P, I32, P,
                                                 ctypes.c_int, I64, I64, I32]),
        "orc_residual_add": (None, [P, P, P, P, I64, ctypes.c_int]),
        "orc_weighted_silu_mul_bounded": (ctypes.c_int, [P, P, P, I64, I64, I64]),
        "orc_epilogue_chain": (ctypes.c_int, [P, P, I64, P, I32, P, P, P, I64, I64, I32,
                                              ctypes.c_int, P, P]),
        "orc_ordered_reduce_scatter_v": (ctypes.c_int, [P, I32, I32, P, I32, I64, I64, I64,
                                                        ctypes.c_int, P, ctypes.c_int]),
        "orc_unpermute_reduce_scatter": (ctypes.c_int, [P, ctypes.c_int, I64, P, I32, I64, I32,
                                                        I32, I32, P, ctypes.c_int, P, P,
                                                        ctypes.c_int, I64, I64]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _lib():
    global _LIB
    with _LOCK:
        if _LIB is None:
            build()
            _LIB = load(_LIB_PATH)
    return _LIB


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def _storage_np(dt):
    return np.float32 if dt == F32 else np.uint16


# ------------------------------------------------------------ scalar dtypes

def bf16_from_f32(values) -> np.ndarray:
    """Round fp32 values to bf16 bits (RNE), elementwise."""
    lib = _lib()
    v = np.asarray(values, dtype=np.float32).ravel()
    return np.array([lib.orc_bf16_from_f32(float(x)) for x in v], dtype=np.uint16)


def f32_from_bf16(bits) -> np.ndarray:
    lib = _lib()
    b = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.orc_f32_from_bf16(int(x)) for x in b], dtype=np.float32)


def f16_from_f32(values) -> np.ndarray:
    lib = _lib()
    v = np.asarray(values, dtype=np.float32).ravel()
    return np.array([lib.orc_f16_from_f32(float(x)) for x in v], dtype=np.uint16)


def f32_from_f16(bits) -> np.ndarray:
    lib = _lib()
    b = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.orc_f32_from_f16(int(x)) for x in b], dtype=np.float32)


# -------------------------------------------------------------- the ops

def swiglu_clamped_fwd(x: np.ndarray, probs: np.ndarray, limit: float, dt: int = BF16):
    """x: [rows, 2*inter] in dtype dt (uint16 bits for bf16/fp16, float32 for fp32);
    probs: float32 [rows] or [rows, 1].  Returns y [rows, inter] in dt."""
    x = _c(x, _storage_np(dt))
    rows, two_i = x.shape
    inter = two_i // 2
    probs = _c(np.asarray(probs, np.float32).reshape(rows), np.float32)
    y = np.empty((rows, inter), _storage_np(dt))
    _lib().orc_swiglu_clamped_fwd_dt(_p(x), _p(probs), _p(y), rows, inter, two_i, inter,
                                     float(limit), dt)
    return y


def swiglu_clamped_bwd(x, probs, grad_y, limit, dt: int = BF16):
    """Returns (grad_x [rows, 2*inter] in dt, grad_probs float64 [rows],
    grad_probs_abs float64 [rows])."""
    x = _c(x, _storage_np(dt))
    rows, two_i = x.shape
    inter = two_i // 2
    probs = _c(np.asarray(probs, np.float32).reshape(rows), np.float32)
    grad_y = _c(grad_y, _storage_np(dt))
    assert grad_y.shape == (rows, inter)
    gx = np.empty((rows, two_i), _storage_np(dt))
    gp = np.empty(rows, np.float64)
    ga = np.empty(rows, np.float64)
    _lib().orc_swiglu_clamped_bwd_dt(_p(x), _p(probs), _p(grad_y), _p(gx), _p(gp), _p(ga),
                                     rows, inter, two_i, inter, two_i, float(limit), dt)
    return gx, gp, ga


def swiglu_clamped_fwd_f64(g, u, p, limit) -> np.ndarray:
    g = _c(np.asarray(g, np.float64).ravel(), np.float64)
    u = _c(np.asarray(u, np.float64).ravel(), np.float64)
    p = _c(np.asarray(p, np.float64).ravel(), np.float64)
    y = np.empty_like(g)
    _lib().orc_swiglu_clamped_fwd_f64(_p(g), _p(u), _p(p), _p(y), g.size, float(limit))
    return y


def router_weight_fwd(x, x_dt, probs, out_dt, p_dt=F32):
    """probs: [rows] or [rows, 1] in dtype p_dt (uint16 bits for bf16/fp16)."""
    x = _c(x, _storage_np(x_dt))
    rows, hidden = x.shape
    probs = _c(np.asarray(probs).reshape(rows), _storage_np(p_dt))
    out = np.empty((rows, hidden), _storage_np(out_dt))
    _lib().orc_router_weight_fwd_p(_p(x), x_dt, _p(probs), p_dt, _p(out), out_dt, rows, hidden)
    return out


def router_weight_bwd(grad_out, g_dt, x, x_dt, probs, p_dt=F32):
    """x may be None (forward did not save x).  Returns (grad_x, grad_probs f64
    or None, grad_probs_abs f64 or None); grad_probs is the unrounded sum."""
    grad_out = _c(grad_out, _storage_np(g_dt))
    rows, hidden = grad_out.shape
    x = _c(x, _storage_np(x_dt))
    probs = _c(np.asarray(probs).reshape(rows), _storage_np(p_dt))
    gx = np.empty((rows, hidden), _storage_np(x_dt))
    gp = np.empty(rows, np.float64) if x is not None else None
    ga = np.empty(rows, np.float64) if x is not None else None
    _lib().orc_router_weight_bwd_p(_p(grad_out), g_dt, _p(x), x_dt, _p(probs), p_dt, _p(gx),
                                   _p(gp), _p(ga), rows, hidden)
    return gx, gp, ga


def act_with_probs_permuted(act, x, out_init, permutation_map, n_used, probs, width,
                            clamp_scale=1.0, zero_padding=False):
    """x: uint16 [max_rows, width or 2*width]; out_init: uint16 [max_rows, width]
    (its contents stand for whatever the output buffer held before the call).
    Returns (out, error_bits)."""
    x = _c(x, np.uint16)
    out = np.array(out_init, dtype=np.uint16, copy=True)
    max_rows = out.shape[0]
    pm = _c(permutation_map, np.int32)
    probs = _c(np.asarray(probs, np.float32).ravel(), np.float32)
    err = _lib().orc_act_with_probs_permuted(act, _p(x), _p(out), _p(pm), int(n_used),
                                             _p(probs), probs.size, max_rows, width,
                                             float(clamp_scale), int(bool(zero_padding)))
    return out, err


def unpermute_ordered(expert_output, in_dt, inverse_map, valid_tokens, out_init, out_dt):
    """expert_output [max_rows, hidden]; inverse_map int32 [tokens, E];
    out_init [tokens, hidden] (prior contents).  Returns (out, error_bits)."""
    eo = _c(expert_output, _storage_np(in_dt))
    max_rows, hidden = eo.shape
    inv = _c(inverse_map, np.int32)
    tokens, n_exp = inv.shape
    out = np.array(out_init, dtype=_storage_np(out_dt), copy=True)
    assert out.shape == (tokens, hidden)
    err = _lib().orc_unpermute_ordered(_p(eo), in_dt, max_rows, _p(inv), int(valid_tokens),
                                       _p(out), out_dt, tokens, hidden, n_exp)
    return out, err


def residual_add(expert_output, shared_expert_output, residual, dt):
    st = _storage_np(dt)
    e = _c(expert_output, st)
    s = _c(shared_expert_output, st)
    r = _c(residual, st)
    assert e.shape == s.shape == r.shape
    out = np.empty_like(r)
    _lib().orc_residual_add(_p(e), _p(s), _p(r), _p(out), e.size, dt)
    return out


def weighted_silu_mul_bounded(y, weights, out_init, bound_elems):
    """y: uint16 [rows, 2*half_n]; weights float32 [rows]; out_init uint16
    [rows, half_n] (prior contents).  Returns (out, error_bits)."""
    y = _c(y, np.uint16)
    rows, two_h = y.shape
    half_n = two_h // 2
    w = _c(np.asarray(weights, np.float32).ravel(), np.float32)
    out = np.array(out_init, dtype=np.uint16, copy=True)
    assert out.shape == (rows, half_n) and w.size == rows
    err = _lib().orc_weighted_silu_mul_bounded(_p(y), _p(w), _p(out), int(bound_elems), rows,
                                               half_n)
    return out, err


def epilogue_chain(expert_output, row_probs, inverse_map, valid_tokens, shared, residual,
                   out_init, dt):
    """The materialised chain router-weight multiply -> ordered unpermute ->
    residual add.  Returns (out, error_bits)."""
    st = _storage_np(dt)
    eo = _c(expert_output, st)
    max_rows, hidden = eo.shape
    rp = _c(np.asarray(row_probs, np.float32).ravel(), np.float32)
    inv = _c(inverse_map, np.int32)
    tokens, n_exp = inv.shape
    sh = _c(shared, st)
    rs = _c(residual, st)
    out = np.array(out_init, dtype=st, copy=True)
    scratch = np.empty((max_rows, hidden), st)
    routed = np.zeros((tokens, hidden), st)
    err = _lib().orc_epilogue_chain(_p(eo), _p(rp), max_rows, _p(inv), int(valid_tokens), _p(sh),
                                    _p(rs), _p(out), tokens, hidden, n_exp, dt, _p(scratch),
                                    _p(routed))
    return out, err


def ordered_reduce_scatter_v(inputs, in_dt, rank, rank_token_offset, ep_tokens, out_init,
                             out_dt):
    """inputs: list of `world` [capacity_rows, hidden] arrays (uint16 bits for
    bf16/fp16), one per rank in rank order; out_init: [local_tokens, hidden]
    (its contents stand for the output buffer before the call).
    Returns (out, error_bits)."""
    st = _storage_np(in_dt)
    ins = [_c(a, st) for a in inputs]
    capacity, hidden = ins[0].shape
    if any(a.shape != (capacity, hidden) for a in ins):
        raise ValueError("every rank's buffer must have the same shape")
    ptrs = (ctypes.c_void_p * len(ins))(*[a.ctypes.data for a in ins])
    offs = _c(np.asarray(rank_token_offset, np.int32).ravel(), np.int32)
    if offs.size != len(ins):
        raise ValueError("one token offset per rank")
    out = np.array(out_init, dtype=_storage_np(out_dt), copy=True)
    local_tokens = out.shape[0]
    err = _lib().orc_ordered_reduce_scatter_v(ctypes.cast(ptrs, ctypes.c_void_p), len(ins),
                                              int(rank), _p(offs), int(ep_tokens), capacity,
                                              local_tokens, hidden, in_dt, _p(out), out_dt)
    return out, err


def unpermute_reduce_scatter(expert_outputs, eo_dt, inverse_maps, ep_tokens, rank,
                             rank_token_offset, partial_dt, out_init, out_dt):
    """expert_outputs: list of `world` [max_rows, hidden] arrays (one per rank,
    rank order); inverse_maps: list of int32 [capacity_rows, E] arrays over the
    token rows of all ranks; out_init: [local_tokens, hidden] (prior contents).
    Returns (out, error_bits)."""
    st = _storage_np(eo_dt)
    eos = [_c(a, st) for a in expert_outputs]
    max_rows, hidden = eos[0].shape
    invs = [_c(a, np.int32) for a in inverse_maps]
    capacity, n_exp = invs[0].shape
    if any(a.shape != (max_rows, hidden) for a in eos) or \
            any(a.shape != (capacity, n_exp) for a in invs) or len(eos) != len(invs):
        raise ValueError("one [max_rows, hidden] block and one [capacity, E] map per rank")
    world = len(eos)
    eo_ptrs = (ctypes.c_void_p * world)(*[a.ctypes.data for a in eos])
    inv_ptrs = (ctypes.c_void_p * world)(*[a.ctypes.data for a in invs])
    offs = _c(np.asarray(rank_token_offset, np.int32).ravel(), np.int32)
    out = np.array(out_init, dtype=_storage_np(out_dt), copy=True)
    partials = np.zeros(world * capacity * hidden, _storage_np(partial_dt))
    err = _lib().orc_unpermute_reduce_scatter(
        ctypes.cast(eo_ptrs, ctypes.c_void_p), eo_dt, max_rows,
        ctypes.cast(inv_ptrs, ctypes.c_void_p), n_exp, capacity, int(ep_tokens), world,
        int(rank), _p(offs), partial_dt, _p(partials), _p(out), out_dt, out.shape[0], hidden)
    return out, err
