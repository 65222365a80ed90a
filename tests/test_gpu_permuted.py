"""Parity of the batch-invariant permuted activation and of the fixed-order
unpermute with the CPU oracle (gpu).

SQRELU, padding, untouched rows and the unpermute are bit-exact; SQRELU_CLAMP
and SWIGLU are within 1 bf16 ulp (tanh / exp implementations differ).
"""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_epilogue_b200 import _abi, inputs, ops
from tests._util import assert_bits_equal, assert_within_ulp16, bits

pytestmark = pytest.mark.gpu

ACTS = [(_abi.MOE_ACT_SQRELU, oracle.SQRELU, 0), (_abi.MOE_ACT_SQRELU_CLAMP, oracle.SQRELU_CLAMP, 1),
        (_abi.MOE_ACT_SWIGLU, oracle.SWIGLU, 1)]
CANARY = 0x1234


def _run_act(dev, act, rt, x, width, scale, zero_padding, n_used=None, pmap=None, err=None):
    out = torch.full((rt.max_rows, width), 0, dtype=torch.int16, device=dev).fill_(CANARY) \
        .view(torch.bfloat16)
    nu = torch.tensor([rt.n_used if n_used is None else n_used], dtype=torch.int32, device=dev)
    pm = (rt.permutation_map if pmap is None else pmap).to(dev)
    ops.act_with_probs_permuted(act, x.to(dev), pm, nu, rt.probs.to(dev), scale, zero_padding,
                                out=out, dev_err=err)
    torch.cuda.synchronize()
    return bits(out)


@pytest.mark.parametrize("act,oact,tol", ACTS)
@pytest.mark.parametrize("zero_padding", [False, True])
@pytest.mark.parametrize("tokens,top_k,experts,align,width", [
    (12, 2, 4, 4, 24), (100, 4, 8, 16, 1001), (257, 8, 16, 128, 1536)])
def test_act_permuted_parity(cuda_device, act, oact, tol, zero_padding, tokens, top_k, experts,
                             align, width):
    rt = inputs.routing(tokens, top_k, experts, align, seed=tokens)
    x = inputs.permuted_activation_input(rt, width, swiglu=(oact == oracle.SWIGLU), seed=tokens + 1)
    got = _run_act(cuda_device, act, rt, x, width, 7.0, zero_padding)
    ref, err = oracle.act_with_probs_permuted(oact, bits(x), np.full((rt.max_rows, width), CANARY,
                                                                     np.uint16),
                                              bits(rt.permutation_map), rt.n_used, bits(rt.probs),
                                              width, 7.0, zero_padding)
    assert err == 0
    if tol == 0:
        assert_bits_equal(got, ref, "act")
    else:
        assert_within_ulp16(got, ref, tol, what="act")
        # padding / untouched rows are exact whatever the activation
        dead = bits(rt.permutation_map) < 0
        assert_bits_equal(got[dead], ref[dead], "padding rows")


@pytest.mark.parametrize("act,oact,tol", ACTS)
def test_act_permuted_full_workload_whole_tensor(cuda_device, act, oact, tol):
    """8192 tokens, top-8 of 64 experts, rows padded to 128 per expert
    (max_rows 73728), hidden 1536 / ffn 1536, zero padding on: every row of
    the output against the oracle (live rows, padding rows, untouched tail)."""
    rt = inputs.routing(8192, 8, 64, 128, seed=0)
    width = 1536
    x = inputs.permuted_activation_input(rt, width, swiglu=(oact == oracle.SWIGLU), seed=1)
    got = _run_act(cuda_device, act, rt, x, width, 7.0, True)
    ref, err = oracle.act_with_probs_permuted(oact, bits(x), np.full((rt.max_rows, width), CANARY,
                                                                     np.uint16),
                                              bits(rt.permutation_map), rt.n_used, bits(rt.probs),
                                              width, 7.0, True)
    assert err == 0
    if tol == 0:
        assert_bits_equal(got, ref, "act")
    else:
        assert_within_ulp16(got, ref, tol, what="act")
    pm = bits(rt.permutation_map)
    assert (got[rt.n_used:] == CANARY).all()
    assert (got[:rt.n_used][pm[:rt.n_used] < 0] == 0).all()


def _placed(t, dev, offset_elems):
    """t copied to the device at an element offset inside a larger buffer."""
    flat = torch.empty(t.numel() + offset_elems, dtype=t.dtype, device=dev)
    v = flat[offset_elems:].view(t.shape)
    v.copy_(t.to(dev))
    return v


# (width, x offset, out offset) in elements: the flat 32-byte kernel (width a
# multiple of 16, both bases 32-byte aligned), the warp-per-row 16-byte kernel
# (width 8 mod 16, or a base only 16-byte aligned) and the per-element kernel
# (a base off 16-byte alignment).
LAYOUTS = [(1536, 0, 0), (48, 0, 0), (16, 0, 0), (1544, 0, 0), (1536, 8, 0), (1536, 0, 8),
           (1536, 1, 0)]


@pytest.mark.parametrize("act,oact,tol", ACTS)
@pytest.mark.parametrize("zero_padding", [False, True])
@pytest.mark.parametrize("width,x_off,out_off", LAYOUTS)
def test_act_permuted_layouts(cuda_device, act, oact, tol, zero_padding, width, x_off, out_off):
    """Every kernel the layout selects, on a ragged routing (300 tokens, top-3 of
    7 experts, rows padded to 16) with the live-row bound cut short, against
    the oracle; untouched rows keep their canary."""
    rt = inputs.routing(300, 3, 7, 16, seed=width + x_off)
    n_used = rt.n_used - 5
    x = inputs.permuted_activation_input(rt, width, swiglu=(oact == oracle.SWIGLU), seed=width)
    canary = torch.full((rt.max_rows, width), CANARY, dtype=torch.int16).view(torch.bfloat16)
    out = _placed(canary, cuda_device, out_off)
    ops.act_with_probs_permuted(act, _placed(x, cuda_device, x_off),
                                rt.permutation_map.to(cuda_device),
                                torch.tensor([n_used], dtype=torch.int32, device=cuda_device),
                                rt.probs.to(cuda_device), 7.0, zero_padding, out=out)
    torch.cuda.synchronize()
    ref, err = oracle.act_with_probs_permuted(oact, bits(x), bits(canary),
                                              bits(rt.permutation_map), n_used, bits(rt.probs),
                                              width, 7.0, zero_padding)
    assert err == 0
    got = bits(out)
    if tol == 0:
        assert_bits_equal(got, ref, "act")
    else:
        assert_within_ulp16(got, ref, tol, what="act")
    assert (got[n_used:] == CANARY).all()


@pytest.mark.parametrize("act", [a for a, _, _ in ACTS])
def test_act_permuted_flat_kernel_batch_invariant(cuda_device, act):
    """The flat kernel's grid and stride follow max_rows: the same live rows in
    a buffer of 3x the rows (123 against 369 CTAs, so every chunk falls at
    another stride phase) give the same bits."""
    rt = inputs.routing(100, 2, 8, 16, seed=11)
    width = 1536
    x = inputs.permuted_activation_input(rt, width, swiglu=act == _abi.MOE_ACT_SWIGLU, seed=12)
    small = _run_act(cuda_device, act, rt, x, width, 7.0, True)
    R = rt.max_rows
    big_x = torch.zeros((3 * R,) + tuple(x.shape[1:]), dtype=x.dtype)
    big_x[:R] = x
    big_pm = torch.full((3 * R,), -1, dtype=torch.int32)
    big_pm[:R] = rt.permutation_map
    out = torch.full((3 * R, width), CANARY, dtype=torch.int16, device=cuda_device) \
        .view(torch.bfloat16)
    ops.act_with_probs_permuted(act, big_x.to(cuda_device), big_pm.to(cuda_device),
                                torch.tensor([rt.n_used], dtype=torch.int32, device=cuda_device),
                                rt.probs.to(cuda_device), 7.0, True, out=out)
    torch.cuda.synchronize()
    got = bits(out)
    assert_bits_equal(got[:R], small, "same rows, larger buffer")
    assert (got[R:] == CANARY).all()


def test_act_permuted_bad_metadata_sets_error_bits(cuda_device):
    rt = inputs.routing(40, 2, 4, 8, seed=3)
    width = 16
    x = inputs.permuted_activation_input(rt, width, swiglu=False, seed=4)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got = _run_act(cuda_device, _abi.MOE_ACT_SQRELU, rt, x, width, 1.0, True,
                   n_used=rt.max_rows + 100, err=err)
    assert int(err) & _abi.MOE_DEVERR_COUNT
    # clamped to max_rows: rows past the old n_used are padding (map < 0) -> zero-filled
    assert (got[rt.n_used:] == 0).all()
    pm = rt.permutation_map.clone()
    live = torch.nonzero(pm >= 0).flatten()
    pm[live[0]] = 1 << 30
    err.zero_()
    got = _run_act(cuda_device, _abi.MOE_ACT_SQRELU, rt, x, width, 1.0, True, pmap=pm, err=err)
    assert int(err) == _abi.MOE_DEVERR_MAP
    assert (got[int(live[0])] == CANARY).all()
    err.zero_()
    _run_act(cuda_device, _abi.MOE_ACT_SQRELU, rt, x, width, 1.0, True, n_used=-5, err=err)
    assert int(err) == _abi.MOE_DEVERR_COUNT


# ------------------------------------------------------------------ unpermute

ODT = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}


def _run_unpermute(dev, rt, eo, out_dtype, valid, inv=None, err=None):
    out = torch.full((rt.tokens, eo.shape[1]), 3.0, dtype=out_dtype, device=dev)
    vt = torch.tensor([valid], dtype=torch.int32, device=dev)
    ops.unpermute_ordered(eo.to(dev), (rt.inverse_map if inv is None else inv).to(dev), vt, out,
                          dev_err=err)
    torch.cuda.synchronize()
    return bits(out)


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32, torch.float16])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32, torch.float16])
@pytest.mark.parametrize("tokens,top_k,experts,align,hidden,valid", [
    (50, 2, 4, 4, 72, 50), (300, 8, 64, 16, 1001, 290), (129, 6, 10, 128, 4096, 100),
    (200, 4, 100, 8, 264, 200), (70, 2, 65, 4, 16, 69), (3000, 8, 64, 16, 512, 2999),
    (90, 5, 12, 4, 48, 90)])
def test_unpermute_bitwise(cuda_device, in_dtype, out_dtype, tokens, top_k, experts, align, hidden,
                           valid):
    rt = inputs.routing(tokens, top_k, experts, align, seed=hidden)
    eo = inputs.expert_output_input(rt, hidden, dtype=in_dtype, seed=hidden + 1)
    got = _run_unpermute(cuda_device, rt, eo, out_dtype, valid)
    init = bits(torch.full((tokens, hidden), 3.0, dtype=out_dtype))
    ref, err = oracle.unpermute_ordered(bits(eo), ODT[in_dtype], bits(rt.inverse_map), valid, init,
                                        ODT[out_dtype])
    assert err == 0
    assert_bits_equal(got, ref, "unpermute", kind="f16" if out_dtype == torch.float16 else "bf16")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_unpermute_full_workload_bitwise(cuda_device, out_dtype):
    """8192 tokens x top-8 of 64 experts, hidden 4096: the whole output."""
    rt = inputs.routing(8192, 8, 64, 128, seed=0)
    eo = inputs.expert_output_input(rt, 4096, seed=2)
    got = _run_unpermute(cuda_device, rt, eo, out_dtype, rt.tokens)
    init = bits(torch.full((rt.tokens, 4096), 3.0, dtype=out_dtype))
    ref, _ = oracle.unpermute_ordered(bits(eo), oracle.BF16, bits(rt.inverse_map), rt.tokens, init,
                                      ODT[out_dtype])
    assert_bits_equal(got, ref, "unpermute")


@pytest.mark.parametrize("hidden", [8, 16])
def test_unpermute_order_witness_and_bad_entries(cuda_device, hidden):
    # contributions 1, 2^24, -2^24 in expert order 0, 1, 2: fp32 gives 0, not 1
    # (hidden 8: 16-byte loads; 16: 32-byte loads)
    rt = inputs.Routing(2, 3, 3, 1, 3, 3, torch.tensor([0, 1, 2], dtype=torch.int32),
                        torch.tensor([[0, 1, 2], [2, 1, 0]], dtype=torch.int32),
                        torch.ones(6), torch.tensor([2, 2, 2]))
    eo = torch.tensor([[1.0] * hidden, [2.0 ** 24] * hidden, [-(2.0 ** 24)] * hidden],
                      dtype=torch.bfloat16)
    got = _run_unpermute(cuda_device, rt, eo, torch.float32, 2)
    assert (got[0] == 0.0).all() and (got[1] == 1.0).all()
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    inv = rt.inverse_map.clone()
    inv[0, 1] = 99
    got = _run_unpermute(cuda_device, rt, eo, torch.float32, 5, inv=inv, err=err)
    assert int(err) == _abi.MOE_DEVERR_COUNT | _abi.MOE_DEVERR_INVERSE
    assert (got[0] == 1.0 - 2.0 ** 24).all()


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("eo_off_bytes,out_off_bytes", [(0, 0), (16, 0), (0, 16), (2, 0)])
def test_unpermute_layouts(cuda_device, out_dtype, eo_off_bytes, out_off_bytes):
    """32-byte aligned bases (32-byte loads), 16-byte aligned ones (16-byte
    loads) and an unaligned input (the per-element kernel), hidden 4096."""
    rt = inputs.routing(257, 8, 64, 16, seed=21)
    hidden = 4096
    eo = inputs.expert_output_input(rt, hidden, seed=22)
    e_off = eo_off_bytes // 2
    o_off = out_off_bytes // (2 if out_dtype == torch.bfloat16 else 4)
    flat_e = torch.empty(eo.numel() + e_off, dtype=eo.dtype, device=cuda_device)
    eo_d = flat_e[e_off:].view(eo.shape)
    eo_d.copy_(eo.to(cuda_device))
    flat_o = torch.full((rt.tokens * hidden + o_off,), 3.0, dtype=out_dtype, device=cuda_device)
    out = flat_o[o_off:].view(rt.tokens, hidden)
    vt = torch.tensor([rt.tokens - 3], dtype=torch.int32, device=cuda_device)
    ops.unpermute_ordered(eo_d, rt.inverse_map.to(cuda_device), vt, out)
    torch.cuda.synchronize()
    init = bits(torch.full((rt.tokens, hidden), 3.0, dtype=out_dtype))
    ref, err = oracle.unpermute_ordered(bits(eo), oracle.BF16, bits(rt.inverse_map),
                                        rt.tokens - 3, init, ODT[out_dtype])
    assert err == 0
    assert_bits_equal(bits(out), ref, "unpermute")


def test_unpermute_batch_invariant(cuda_device):
    """A token's bits do not depend on the other tokens: shuffling the rest of
    the batch (and its size) leaves them unchanged."""
    rt = inputs.routing(512, 8, 64, 16, seed=5)
    eo = inputs.expert_output_input(rt, 2048, seed=6)
    full = _run_unpermute(cuda_device, rt, eo, torch.bfloat16, rt.tokens)
    perm = torch.randperm(rt.tokens, generator=torch.Generator().manual_seed(7))
    sub = perm[:37]
    rt2 = inputs.Routing(37, 8, 64, 16, rt.max_rows, rt.n_used, rt.permutation_map,
                         rt.inverse_map[sub].contiguous(), rt.probs, rt.counts)
    part = _run_unpermute(cuda_device, rt2, eo, torch.bfloat16, 37)
    assert_bits_equal(part, full[sub.numpy()], "batch invariance")


@pytest.mark.parametrize("act,oact,tol", ACTS)
@pytest.mark.parametrize("scale", [1.0, 7.0, 30.0])
def test_act_permuted_special_values(cuda_device, act, oact, tol, scale):
    """NaN, +-inf, +-0, tiny and huge inputs, and values on both sides of the
    switch between the two tanh forms (y = x/s around 1/32)."""
    vals = [float("nan"), float("inf"), -float("inf"), 0.0, -0.0, 1e-30, -1e-30, 1e-39, 3e38,
            -3e38, 1e30, scale / 32, scale / 32 * 1.01, scale / 32 * 0.99, -scale / 32, 0.5, -0.5,
            2.0, 9.0, 44.0 * scale, 100.0 * scale, -88.5, -87.0, 20.0]
    width = 8 * ((len(vals) + 7) // 8)
    row = torch.tensor(vals + [1.0] * (width - len(vals)), dtype=torch.bfloat16)
    rows = 4
    cols = 2 * width if oact == oracle.SWIGLU else width
    x = torch.zeros(rows, cols, dtype=torch.bfloat16)
    for r in range(rows):
        x[r, :width] = row.roll(r)
        if cols > width:
            x[r, width:] = row.roll(-r)
    rt = inputs.Routing(rows, 1, 1, 1, rows, rows, torch.arange(rows, dtype=torch.int32),
                        torch.arange(rows, dtype=torch.int32).reshape(rows, 1),
                        torch.tensor([0.25, 1.0, 0.7, 3.0]), torch.tensor([rows]))
    got = _run_act(cuda_device, act, rt, x, width, scale, True)
    ref, _ = oracle.act_with_probs_permuted(oact, bits(x), np.zeros((rows, width), np.uint16),
                                            bits(rt.permutation_map), rows, bits(rt.probs), width,
                                            scale, True)
    if tol == 0:
        assert_bits_equal(got, ref, "act specials")
    else:
        assert_within_ulp16(got, ref, tol, what="act specials")
