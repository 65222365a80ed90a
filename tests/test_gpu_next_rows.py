"""Parity of the device-bounded weighted SwiGLU and of the fused epilogue chain
with the CPU oracle (gpu).

Bounded SwiGLU: within 1 bf16 ulp (exp implementations differ), elements past
the bound untouched, bits independent of the grid size.  Fused chain:
bit-exact against the oracle's materialised chain and against the three
library kernels run one after another.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_epilogue_b200 import _abi, inputs, ops
from tests._util import assert_bits_equal, assert_within_ulp16, bits

pytestmark = pytest.mark.gpu
CANARY = 0x1234


def _bounded_inputs(rows, half_n, seed, sigma=3.0):
    g = torch.Generator().manual_seed(seed)
    y = (torch.randn(rows, 2 * half_n, generator=g) * sigma).to(torch.bfloat16)
    w = torch.rand(rows, generator=g)
    return y, w


def _run_bounded(dev, y, w, bound, num_programs=0, err=None):
    rows, two_h = y.shape
    out = torch.full((rows, two_h // 2), 0, dtype=torch.int16, device=dev).fill_(CANARY) \
        .view(torch.bfloat16)
    b = torch.tensor([bound], dtype=torch.int64, device=dev)
    ops.weighted_silu_mul_bounded(y.to(dev), w.to(dev), b, num_programs=num_programs, out=out,
                                  dev_err=err)
    torch.cuda.synchronize()
    return bits(out)


@pytest.mark.parametrize("rows,half_n,live,extra", [
    (300, 1536, 250, 17), (300, 1536, 300, 0), (64, 1001, 40, 5), (33, 8, 33, 0), (10, 64, 0, 3),
    (5, 2048, 0, 0)])
def test_bounded_parity(cuda_device, rows, half_n, live, extra):
    y, w = _bounded_inputs(rows, half_n, rows + half_n)
    bound = live * half_n + extra
    got = _run_bounded(cuda_device, y, w, bound)
    ref, err = oracle.weighted_silu_mul_bounded(bits(y), bits(w),
                                                np.full((rows, half_n), CANARY, np.uint16), bound)
    assert err == 0
    assert_within_ulp16(got, ref, 1, what="bounded")
    assert (got.reshape(-1)[bound:] == CANARY).all()


def test_bounded_grid_size_cannot_change_bits(cuda_device):
    y, w = _bounded_inputs(777, 512, 5)
    bound = 700 * 512 + 100
    base = _run_bounded(cuda_device, y, w, bound)
    for n in (1, 3, 148, 1184, 5000):
        assert_bits_equal(_run_bounded(cuda_device, y, w, bound, num_programs=n), base,
                          f"num_programs={n}")


def test_bounded_bad_bound_sets_error(cuda_device):
    y, w = _bounded_inputs(8, 16, 6)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got = _run_bounded(cuda_device, y, w, 10 ** 9, err=err)
    assert int(err) == _abi.MOE_DEVERR_COUNT and (got != CANARY).all()
    err.zero_()
    got = _run_bounded(cuda_device, y, w, -4, err=err)
    assert int(err) == _abi.MOE_DEVERR_COUNT and (got == CANARY).all()


def test_bounded_full_size_whole_tensor(cuda_device):
    """65536 rows (8192 tokens x top-8) x half_n 1536, 60000 live rows: every
    live element against the oracle, the rows past the bound untouched."""
    rows, half_n, live = 65536, 1536, 60000
    y, w = _bounded_inputs(rows, half_n, 7)
    got = _run_bounded(cuda_device, y, w, live * half_n)
    ref, err = oracle.weighted_silu_mul_bounded(bits(y)[:live], bits(w)[:live],
                                                np.zeros((live, half_n), np.uint16),
                                                live * half_n)
    assert err == 0
    assert_within_ulp16(got[:live], ref, 1, what="bounded full size")
    assert (got[live:] == CANARY).all()


# ------------------------------------------------------------ fused chain

ODT = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}


def _chain_case(dtype, tokens, top_k, experts, align, hidden, seed):
    rt = inputs.routing(tokens, top_k, experts, align, seed=seed)
    eo = inputs.expert_output_input(rt, hidden, dtype=dtype, seed=seed + 1)
    pm = rt.permutation_map
    row_probs = torch.where(pm >= 0, rt.probs[pm.clamp(min=0).long()], torch.zeros(())).float()
    res = inputs.residual_inputs((tokens, hidden), dtype, seed=seed + 2)
    return rt, eo, row_probs, res["shared_expert_output"], res["residual"]


def _kind(dtype):
    return "f16" if dtype == torch.float16 else "bf16"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("tokens,top_k,experts,align,hidden,valid", [
    (64, 4, 8, 16, 256, 64), (300, 8, 64, 128, 1032, 280), (100, 3, 100, 8, 72, 99),
    (40, 2, 6, 4, 13, 40)])
def test_fused_chain_bitwise(cuda_device, dtype, tokens, top_k, experts, align, hidden, valid):
    rt, eo, rp, sh, rs = _chain_case(dtype, tokens, top_k, experts, align, hidden, hidden)
    init = torch.full((tokens, hidden), 3.0, dtype=dtype)
    out = init.to(cuda_device)
    vt = torch.tensor([valid], dtype=torch.int32, device=cuda_device)
    ops.epilogue_fused(eo.to(cuda_device), rp.to(cuda_device), rt.inverse_map.to(cuda_device), vt,
                       sh.to(cuda_device), rs.to(cuda_device), out=out)
    torch.cuda.synchronize()
    ref, err = oracle.epilogue_chain(bits(eo), bits(rp), bits(rt.inverse_map), valid, bits(sh),
                                     bits(rs), bits(init), ODT[dtype])
    assert err == 0
    assert_bits_equal(bits(out), ref, "fused chain", kind=_kind(dtype))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fused_chain_equals_the_three_library_kernels(cuda_device, dtype):
    """router-weight fwd over the expert rows, then the ordered unpermute, then
    the residual add -- run as three launches -- give the fused kernel's bits,
    including in place (out == residual)."""
    rt, eo, rp, sh, rs = _chain_case(dtype, 512, 8, 64, 128, 2048, 31)
    d = cuda_device
    eo_d, rp_d, inv_d = eo.to(d), rp.to(d), rt.inverse_map.to(d)
    sh_d, rs_d = sh.to(d), rs.to(d)
    vt = torch.tensor([rt.tokens], dtype=torch.int32, device=d)
    w = ops.router_weight_mul_fwd(eo_d, rp_d, dtype)
    routed = torch.empty_like(rs_d)
    ops.unpermute_ordered(w, inv_d, vt, routed)
    chained = ops.residual_add(routed, sh_d, rs_d)
    fused = ops.epilogue_fused(eo_d, rp_d, inv_d, vt, sh_d, rs_d)
    in_place = rs_d.clone()
    ops.epilogue_fused(eo_d, rp_d, inv_d, vt, sh_d, in_place, out=in_place)
    torch.cuda.synchronize()
    assert_bits_equal(bits(fused), bits(chained), "fused vs chained kernels")
    assert_bits_equal(bits(in_place), bits(chained), "in place")


def test_fused_chain_full_workload_whole_tensor(cuda_device):
    """8192 tokens x top-8 of 64 experts, hidden 4096, bf16: every token."""
    rt, eo, rp, sh, rs = _chain_case(torch.bfloat16, 8192, 8, 64, 128, 4096, 41)
    d = cuda_device
    vt = torch.tensor([rt.tokens], dtype=torch.int32, device=d)
    out = ops.epilogue_fused(eo.to(d), rp.to(d), rt.inverse_map.to(d), vt, sh.to(d), rs.to(d))
    torch.cuda.synchronize()
    ref, err = oracle.epilogue_chain(bits(eo), bits(rp), bits(rt.inverse_map), rt.tokens,
                                     bits(sh), bits(rs), np.zeros((rt.tokens, 4096), np.uint16),
                                     oracle.BF16)
    assert err == 0
    assert_bits_equal(bits(out), ref, "fused chain full size")


def test_fused_chain_bad_entries(cuda_device):
    rt, eo, rp, sh, rs = _chain_case(torch.bfloat16, 20, 2, 4, 4, 16, 51)
    d = cuda_device
    inv = rt.inverse_map.clone()
    inv[0, torch.nonzero(inv[0] >= 0)[0, 0]] = rt.max_rows + 7
    err = torch.zeros(1, dtype=torch.int32, device=d)
    vt = torch.tensor([25], dtype=torch.int32, device=d)
    ops.epilogue_fused(eo.to(d), rp.to(d), inv.to(d), vt, sh.to(d), rs.to(d), dev_err=err)
    torch.cuda.synchronize()
    assert int(err) == _abi.MOE_DEVERR_COUNT | _abi.MOE_DEVERR_INVERSE
