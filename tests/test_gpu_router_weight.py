"""Parity of the router-weight multiply kernels with the CPU oracle (gpu).

Forward and grad_x are single fp32 multiplies with one rounding: bit-exact.
grad_probs is a row reduction: within 1e-5 * max(|ref|, sum_h |t_h|).
"""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_epilogue_b200 import _abi, inputs, ops
from tests._util import assert_bits_equal, assert_sum_close, bits

pytestmark = pytest.mark.gpu

ODT = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}
DTYPES = [torch.bfloat16, torch.float16, torch.float32]


@pytest.mark.parametrize("rows,hidden", [(129, 7176), (300, 1001), (1, 8), (7, 3), (2048, 256)])
@pytest.mark.parametrize("x_dtype", DTYPES)
@pytest.mark.parametrize("out_dtype", DTYPES)
def test_router_weight_fwd_bitwise(cuda_device, rows, hidden, x_dtype, out_dtype):
    d = inputs.router_weight_inputs(rows, hidden, seed=rows + hidden)
    x = d["x"].to(x_dtype)
    out = ops.router_weight_mul_fwd(x.to(cuda_device), d["probs"].to(cuda_device), out_dtype)
    torch.cuda.synchronize()
    ref = oracle.router_weight_fwd(bits(x), ODT[x_dtype], bits(d["probs"]), ODT[out_dtype])
    assert_bits_equal(bits(out), ref, "fwd", kind="f16" if out_dtype == torch.float16 else "bf16")


@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("hidden", [4096, 4104, 1004, 12, 7])
@pytest.mark.parametrize("x_shift,out_shift", [(0, 0), (4, 0), (2, 0), (0, 2), (0, 4), (8, 0)])
def test_router_weight_fwd_16bit_to_fp32_layouts(cuda_device, x_dtype, hidden, x_shift,
                                                 out_shift):
    """A 16-bit input scaled into fp32, with rows of 8- or 4-element units
    (hidden % 8 == 0, hidden % 4 == 0) and without, inputs 16-byte (x_shift 8),
    8-byte (4) or 4-byte (2) aligned, and an fp32 output 16- but not 32-byte
    aligned (out_shift 4) or off 16-byte alignment (2): every path gives the
    oracle's bits."""
    rows = 37
    d = inputs.router_weight_inputs(rows, hidden, seed=hidden + x_shift)
    x = d["x"].to(x_dtype)
    xbuf = torch.zeros(rows * hidden + x_shift, dtype=x_dtype, device=cuda_device)
    xd = xbuf[x_shift:].view(rows, hidden)
    xd.copy_(x.to(cuda_device))
    obuf = torch.full((rows * hidden + out_shift,), 7.0, device=cuda_device)
    od = obuf[out_shift:].view(rows, hidden)
    ops.router_weight_mul_fwd(xd, d["probs"].to(cuda_device), torch.float32, out=od)
    torch.cuda.synchronize()
    ref = oracle.router_weight_fwd(bits(x), ODT[x_dtype], bits(d["probs"]), oracle.F32)
    assert_bits_equal(bits(od), ref, "fwd")
    assert (obuf[:out_shift] == 7.0).all()


@pytest.mark.parametrize("rows,hidden", [(129, 7176), (300, 1001), (1, 8), (3000, 40),
                                         (257, 7168), (64, 48), (5, 16), (33, 4096)])
@pytest.mark.parametrize("g_dtype", [torch.bfloat16, torch.float32, torch.float16])
@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("save_x", [True, False])
def test_router_weight_bwd(cuda_device, rows, hidden, g_dtype, x_dtype, save_x):
    d = inputs.router_weight_inputs(rows, hidden, out_dtype=g_dtype, seed=rows * 3 + hidden)
    x = d["x"].to(x_dtype)
    gx, gp = ops.router_weight_mul_bwd(d["grad_out"].to(cuda_device),
                                       x.to(cuda_device) if save_x else None,
                                       d["probs"].to(cuda_device), x_dtype=x_dtype)
    torch.cuda.synchronize()
    gx_ref, gp_ref, gabs = oracle.router_weight_bwd(bits(d["grad_out"]), ODT[g_dtype],
                                                    bits(x) if save_x else None, ODT[x_dtype],
                                                    bits(d["probs"]))
    assert_bits_equal(bits(gx), gx_ref, "grad_x")
    if save_x:
        assert_sum_close(bits(gp).ravel(), gp_ref, gabs, 1e-5, "grad_probs")
    else:
        assert gp is None


@pytest.mark.parametrize("g_off,x_off,gx_off", [(0, 0, 0), (8, 0, 0), (0, 8, 0), (0, 0, 8)])
def test_router_weight_bwd_layouts(cuda_device, g_off, x_off, gx_off):
    """Bases 32-byte aligned (32-byte loads) or only 16-byte aligned (an
    offset of 8 bf16 elements: 16-byte loads), 7168-wide rows."""
    rows, hidden = 200, 7168
    d = inputs.router_weight_inputs(rows, hidden, seed=17)

    def placed(t, off):
        buf = torch.empty(t.numel() + off, dtype=t.dtype, device=cuda_device)
        v = buf[off:].view(t.shape)
        v.copy_(t.to(cuda_device))
        return v

    g, x = placed(d["grad_out"], g_off), placed(d["x"], x_off)
    gx = placed(torch.full((rows, hidden), 5.0, dtype=torch.bfloat16), gx_off)
    gp = torch.empty(rows, dtype=torch.float32, device=cuda_device)
    _abi.moe_router_weight_mul_bwd(g, _abi.MOE_BF16, x, _abi.MOE_BF16,
                                   d["probs"].to(cuda_device), gx, gp, rows, hidden, None)
    torch.cuda.synchronize()
    gx_ref, gp_ref, gabs = oracle.router_weight_bwd(bits(d["grad_out"]), oracle.BF16,
                                                    bits(d["x"]), oracle.BF16, bits(d["probs"]))
    assert_bits_equal(bits(gx), gx_ref, "grad_x")
    assert_sum_close(bits(gp).ravel(), gp_ref, gabs, 1e-5, "grad_probs")


@pytest.mark.parametrize("off", [0, 4])
def test_router_weight_bwd_fp32_grad_without_x(cuda_device, off):
    """fp32 grad_out, x not saved: 32-byte aligned rows (one 32-byte load per
    chunk) and rows only 16-byte aligned (off 4 floats: two 16-byte loads)."""
    rows, hidden = 130, 7168
    d = inputs.router_weight_inputs(rows, hidden, out_dtype=torch.float32, seed=23)
    buf = torch.empty(rows * hidden + off, dtype=torch.float32, device=cuda_device)
    g = buf[off:].view(rows, hidden)
    g.copy_(d["grad_out"].to(cuda_device))
    gx, gp = ops.router_weight_mul_bwd(g, None, d["probs"].to(cuda_device),
                                       x_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    gx_ref, _, _ = oracle.router_weight_bwd(bits(d["grad_out"]), oracle.F32, None, oracle.BF16,
                                            bits(d["probs"]))
    assert gp is None
    assert_bits_equal(bits(gx), gx_ref, "grad_x")


def test_router_weight_unaligned(cuda_device):
    rows, hidden = 33, 64
    d = inputs.router_weight_inputs(rows, hidden, seed=5)
    buf = torch.empty(rows * hidden + 1, dtype=torch.bfloat16, device=cuda_device)
    x = buf[1:].view(rows, hidden)
    x.copy_(d["x"].to(cuda_device))
    p = d["probs"].to(cuda_device)
    out = ops.router_weight_mul_fwd(x, p, torch.float32)
    gx, gp = ops.router_weight_mul_bwd(d["grad_out"].to(cuda_device), x, p)
    torch.cuda.synchronize()
    assert_bits_equal(bits(out), oracle.router_weight_fwd(bits(d["x"]), oracle.BF16,
                                                          bits(d["probs"]), oracle.F32), "fwd")
    gx_ref, gp_ref, gabs = oracle.router_weight_bwd(bits(d["grad_out"]), oracle.BF16,
                                                    bits(d["x"]), oracle.BF16, bits(d["probs"]))
    assert_bits_equal(bits(gx), gx_ref, "grad_x")
    assert_sum_close(bits(gp).ravel(), gp_ref, gabs, 1e-5, "grad_probs")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_router_weight_full_workload_whole_tensor(cuda_device, out_dtype):
    """[16384, 7168] expert outputs, U(0.01, 1) probs: the full launches (fwd
    and both grads, save_x on and off), every element against the oracle."""
    from tests.test_gpu_swiglu import strict_grad_probs_report
    rows, hidden = 16384, 7168
    d = inputs.router_weight_inputs(rows, hidden, out_dtype=out_dtype, seed=0)
    x, p, g = (d[k].to(cuda_device) for k in ("x", "probs", "grad_out"))
    out = ops.router_weight_mul_fwd(x, p, out_dtype)
    gx, gp = ops.router_weight_mul_bwd(g, x, p)
    gx2, _ = ops.router_weight_mul_bwd(g, None, p, x_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    xb, pb, gb = bits(d["x"]), bits(d["probs"]), bits(d["grad_out"])
    assert_bits_equal(bits(out), oracle.router_weight_fwd(xb, oracle.BF16, pb, ODT[out_dtype]),
                      "fwd")
    gx_ref, gp_ref, gabs = oracle.router_weight_bwd(gb, ODT[out_dtype], xb, oracle.BF16, pb)
    assert_bits_equal(bits(gx), gx_ref, "grad_x")
    assert_bits_equal(bits(gx2), gx_ref, "grad_x (x not saved)")
    got = bits(gp).ravel()
    assert_sum_close(got, gp_ref, gabs, 1e-5, "grad_probs")
    rep = strict_grad_probs_report(got, gp_ref, gabs)
    print(f"\ngrad_probs strict relative 1e-5, grad_out {out_dtype}: {rep}")
    assert rep["strict_fail_not_cancelling"] <= rep["rows_not_cancelling"] // 100
    # eager torch on the device computes the same forward bits (the page's definition)
    iv = torch.int16 if out_dtype != torch.float32 else torch.int32
    assert torch.equal((x.float() * p).to(out_dtype).view(iv), out.view(iv))


# Unit roundoff of the probabilities' dtype: grad_probs is the fp32 row sum
# rounded once (RNE) to that dtype.
UNIT_ROUNDOFF = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


@pytest.mark.parametrize("p_dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("rows,hidden", [(129, 7176), (300, 1001), (1, 8), (3000, 40)])
@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float32])
def test_router_weight_low_precision_probs(cuda_device, p_dtype, rows, hidden, x_dtype):
    """Routing probabilities stored in bf16/fp16: out and grad_x bit-exact
    against the oracle; grad_probs in the probabilities' dtype within one
    rounding of it plus the reduction tolerance."""
    d = inputs.router_weight_inputs(rows, hidden, seed=rows + 7 * hidden)
    x = d["x"].to(x_dtype)
    p = d["probs"].to(p_dtype)
    xd, pd, gd = x.to(cuda_device), p.to(cuda_device), d["grad_out"].to(cuda_device)
    out = ops.router_weight_mul_fwd(xd, pd, torch.bfloat16)
    gx, gp = ops.router_weight_mul_bwd(gd, xd, pd)
    gx2, gp2 = ops.router_weight_mul_bwd(gd, None, pd, x_dtype=x_dtype)
    torch.cuda.synchronize()
    assert gp.dtype == p_dtype and gp2 is None
    assert_bits_equal(bits(out), oracle.router_weight_fwd(bits(x), ODT[x_dtype], bits(p),
                                                          oracle.BF16, ODT[p_dtype]), "fwd")
    gx_ref, gp_ref, gabs = oracle.router_weight_bwd(bits(d["grad_out"]), oracle.BF16, bits(x),
                                                    ODT[x_dtype], bits(p), ODT[p_dtype])
    assert_bits_equal(bits(gx), gx_ref, "grad_x")
    assert_bits_equal(bits(gx2), gx_ref, "grad_x (x not saved)")
    got = gp.float().cpu().numpy().ravel().astype(np.float64)
    bound = UNIT_ROUNDOFF[p_dtype] * np.abs(gp_ref) + 1.01e-5 * np.maximum(np.abs(gp_ref), gabs)
    assert (np.abs(got - gp_ref) <= bound).all(), "grad_probs"
    # the 16-bit probabilities widen exactly: same bits as fp32 probabilities of equal value
    out32 = ops.router_weight_mul_fwd(xd, pd.float(), torch.bfloat16)
    torch.cuda.synchronize()
    assert_bits_equal(bits(out32), bits(out), "fwd vs widened fp32 probs")
