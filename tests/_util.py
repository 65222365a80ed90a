"""Comparison helpers shared by the tests (no op arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

from moe_expert_epilogue_b200.inputs import bits, from_bits  # noqa: F401  (re-export)


def is_nan16(b: np.ndarray, kind="bf16") -> np.ndarray:
    b = np.asarray(b, np.uint16)
    if kind == "bf16":
        return ((b & 0x7F80) == 0x7F80) & ((b & 0x007F) != 0)
    return ((b & 0x7C00) == 0x7C00) & ((b & 0x03FF) != 0)


def ord16(b: np.ndarray) -> np.ndarray:
    """Monotone integer image of 16-bit sign-magnitude floats (+0 == -0)."""
    b = np.asarray(b, np.uint16).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def ord32(f: np.ndarray) -> np.ndarray:
    u = np.asarray(f, np.float32).view(np.uint32).astype(np.int64)
    mag = u & 0x7FFFFFFF
    return np.where(u & 0x80000000, -mag, mag)


def ulp_diff16(a, b, kind="bf16"):
    """|ord(a) - ord(b)| with NaN positions required to match (distance 0)."""
    a = np.asarray(a, np.uint16)
    b = np.asarray(b, np.uint16)
    na, nb = is_nan16(a, kind), is_nan16(b, kind)
    if not np.array_equal(na, nb):
        bad = np.argwhere(na != nb)[:5]
        raise AssertionError(f"NaN positions differ, e.g. at {bad.tolist()}")
    d = np.abs(ord16(a) - ord16(b))
    d[na] = 0
    return d


def assert_within_ulp16(got, want, max_ulp=1, kind="bf16", what=""):
    d = ulp_diff16(got, want, kind)
    if d.size and d.max() > max_ulp:
        idx = np.unravel_index(int(d.argmax()), d.shape)
        raise AssertionError(
            f"{what}: {int((d > max_ulp).sum())} elements beyond {max_ulp} ulp; worst "
            f"{int(d.max())} ulp at {idx}: got 0x{int(np.asarray(got)[idx]):04x} "
            f"want 0x{int(np.asarray(want)[idx]):04x}")
    return d


def assert_bits_equal(got, want, what="", kind="bf16"):
    """Bit-exact equality, except that any NaN equals any NaN."""
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, (got.shape, want.shape)
    if got.dtype == np.float32:
        gn, wn = np.isnan(got), np.isnan(want)
        gb, wb = got.view(np.uint32), want.view(np.uint32)
    else:
        gn, wn = is_nan16(got, kind), is_nan16(want, kind)
        gb, wb = got.astype(np.uint16), want.astype(np.uint16)
    if not np.array_equal(gn, wn):
        raise AssertionError(f"{what}: NaN positions differ")
    neq = (gb != wb) & ~gn
    if neq.any():
        idx = tuple(np.argwhere(neq)[0])
        raise AssertionError(f"{what}: {int(neq.sum())} elements differ; first at {idx}: "
                             f"got {gb[idx]!r} want {wb[idx]!r}")


def assert_sum_close(got, ref64, abs64, rtol=1e-5, what=""):
    """Reduction tolerance: |got - ref| <= rtol * max(|ref|, sum_j |t_j|)."""
    got = np.asarray(got, np.float64)
    ref64 = np.asarray(ref64, np.float64)
    bound = rtol * np.maximum(np.abs(ref64), np.asarray(abs64, np.float64))
    err = np.abs(got - ref64)
    bad = err > bound
    if bad.any():
        i = int(np.argmax(err - bound))
        raise AssertionError(f"{what}: {int(bad.sum())} rows beyond tolerance; row {i}: "
                             f"got {got[i]!r} ref {ref64[i]!r} bound {bound[i]!r}")
    return err


def torch_bits(t: torch.Tensor) -> np.ndarray:
    return bits(t)
