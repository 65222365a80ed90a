"""Parity of the fused residual add with the CPU oracle (gpu): bit-exact in
bf16, fp16 and fp32, including in place and on ragged / unaligned sizes."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_epilogue_b200 import inputs, ops
from tests._util import assert_bits_equal, bits

pytestmark = pytest.mark.gpu

ODT = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}
DTYPES = [torch.bfloat16, torch.float16, torch.float32]


def _kind(dt):
    return "f16" if dt == torch.float16 else "bf16"


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", [(37, 129), (1, 7), (1000, 4096), (3, 1)])
def test_residual_add_bitwise(cuda_device, dtype, shape):
    d = inputs.residual_inputs(shape, dtype, seed=shape[0])
    e, s, r = (d[k].to(cuda_device) for k in ("expert_output", "shared_expert_output", "residual"))
    out = ops.residual_add(e, s, r)
    torch.cuda.synchronize()
    ref = oracle.residual_add(*(bits(d[k]) for k in ("expert_output", "shared_expert_output",
                                                     "residual")), ODT[dtype])
    assert_bits_equal(bits(out), ref, "residual add", kind=_kind(dtype))
    # and the eager two-add definition on the device
    assert_bits_equal(bits(r + (e + s)), bits(out), "vs torch", kind=_kind(dtype))


@pytest.mark.parametrize("dtype", DTYPES)
def test_residual_add_in_place_and_unaligned(cuda_device, dtype):
    n = 10007
    d = inputs.residual_inputs((n,), dtype, seed=3)
    ref = oracle.residual_add(*(bits(d[k]) for k in ("expert_output", "shared_expert_output",
                                                     "residual")), ODT[dtype])
    e, s, r = (d[k].to(cuda_device) for k in ("expert_output", "shared_expert_output", "residual"))
    ops.residual_add(e, s, r, out=r)                     # in place
    torch.cuda.synchronize()
    assert_bits_equal(bits(r), ref, "in place", kind=_kind(dtype))
    buf = torch.empty(n + 1, dtype=dtype, device=cuda_device)
    rr = buf[1:]
    rr.copy_(d["residual"].to(cuda_device))
    out = ops.residual_add(e, s, rr)                     # residual not 16-byte aligned
    torch.cuda.synchronize()
    assert_bits_equal(bits(out), ref, "unaligned", kind=_kind(dtype))


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("which", [0, 1, 2, 3])
def test_residual_add_16_byte_aligned(cuda_device, dtype, which):
    """One of the four tensors 16- but not 32-byte aligned (the 16-byte
    stream instead of the 32-byte one), 10007 elements."""
    n = 10007
    shift = 16 // torch.empty((), dtype=dtype).element_size()
    d = inputs.residual_inputs((n,), dtype, seed=9)
    names = ("expert_output", "shared_expert_output", "residual")
    ref = oracle.residual_add(*(bits(d[k]) for k in names), ODT[dtype])
    ts = []
    for i, k in enumerate(names):
        off = shift if i == which else 0
        buf = torch.empty(n + off, dtype=dtype, device=cuda_device)
        ts.append(buf[off:])
        ts[-1].copy_(d[k].to(cuda_device))
    obuf = torch.empty(n + (shift if which == 3 else 0), dtype=dtype, device=cuda_device)
    out = obuf[shift if which == 3 else 0:]
    ops.residual_add(*ts, out=out)
    torch.cuda.synchronize()
    assert_bits_equal(bits(out), ref, "16-byte aligned", kind=_kind(dtype))


@pytest.mark.parametrize("dtype", DTYPES)
def test_residual_add_full_workload_whole_tensor(cuda_device, dtype):
    """[32768, 7168], all inputs N(0,1): the full launch, every element
    against the oracle."""
    shape = (32768, 7168)
    d = inputs.residual_inputs(shape, dtype, seed=0)
    e, s, r = (d[k].to(cuda_device) for k in ("expert_output", "shared_expert_output", "residual"))
    out = ops.residual_add(e, s, r)
    torch.cuda.synchronize()
    ref = oracle.residual_add(*(bits(d[k]) for k in
                                ("expert_output", "shared_expert_output", "residual")), ODT[dtype])
    assert_bits_equal(bits(out), ref, "residual add", kind=_kind(dtype))
    assert_bits_equal(bits(out), bits(r + (e + s)), "whole tensor vs torch", kind=_kind(dtype))


def test_epilogue_chain_router_weight_then_residual(cuda_device):
    """The chained epilogue pass: e = router-weight forward of an expert output,
    then residual + (e + shared); each step bit-exact against the oracle."""
    rows, hidden = 512, 7168
    rw = inputs.router_weight_inputs(rows, hidden, seed=8)
    res = inputs.residual_inputs((rows, hidden), torch.bfloat16, seed=9)
    x, p = rw["x"].to(cuda_device), rw["probs"].to(cuda_device)
    e = ops.router_weight_mul_fwd(x, p, torch.bfloat16)
    s, r = res["shared_expert_output"].to(cuda_device), res["residual"].to(cuda_device)
    out = ops.residual_add(e, s, r)
    torch.cuda.synchronize()
    e_ref = oracle.router_weight_fwd(bits(rw["x"]), oracle.BF16, bits(rw["probs"]), oracle.BF16)
    ref = oracle.residual_add(e_ref, bits(res["shared_expert_output"]), bits(res["residual"]),
                              oracle.BF16)
    assert_bits_equal(bits(out), ref, "chain")
