"""Empty and degenerate inputs through the public front end (gpu).

Zero rows, zero columns, zero live rows / valid tokens, tokens routed to no
local expert: every call succeeds, writes nothing it should not, and the
empty reductions give +0 (the sum over no terms)."""
import numpy as np
import pytest
import torch

from moe_expert_epilogue_b200 import ops
from tests._util import bits

pytestmark = pytest.mark.gpu
NAN = float("nan")


def test_swiglu_empty(cuda_device):
    d = cuda_device
    y = ops.swiglu_clamped_fwd(torch.zeros(0, 64, dtype=torch.bfloat16, device=d),
                               torch.zeros(0, 1, device=d), 7.0)
    gx, gp = ops.swiglu_clamped_bwd(torch.zeros(0, 64, dtype=torch.bfloat16, device=d),
                                    torch.zeros(0, 1, device=d),
                                    torch.zeros(0, 32, dtype=torch.bfloat16, device=d), 7.0)
    assert y.shape == (0, 32) and gx.shape == (0, 64) and gp.shape == (0, 1)
    # inter = 0: no output elements, and grad_probs is the empty sum +0
    x0 = torch.zeros(5, 0, dtype=torch.bfloat16, device=d)
    p = torch.rand(5, 1, device=d)
    ops.swiglu_clamped_fwd(x0, p, 7.0)
    gp = torch.full((5, 1), NAN, device=d)
    ops.swiglu_clamped_bwd(x0, p, torch.zeros(5, 0, dtype=torch.bfloat16, device=d), 7.0,
                           grad_probs=gp)
    torch.cuda.synchronize()
    assert (bits(gp).view(np.uint32) == 0).all()


def test_router_weight_empty(cuda_device):
    d = cuda_device
    out = ops.router_weight_mul_fwd(torch.zeros(0, 16, dtype=torch.bfloat16, device=d),
                                    torch.zeros(0, 1, device=d))
    assert out.shape == (0, 16)
    x0 = torch.zeros(6, 0, dtype=torch.bfloat16, device=d)
    p = torch.rand(6, 1, device=d)
    ops.router_weight_mul_fwd(x0, p)
    gp = torch.full((6, 1), NAN, device=d)
    gx, gp = ops.router_weight_mul_bwd(x0, x0, p, grad_probs=gp)
    torch.cuda.synchronize()
    assert gx.shape == (6, 0) and (bits(gp).view(np.uint32) == 0).all()


def test_permuted_and_unpermute_nothing_live(cuda_device):
    d = cuda_device
    x = torch.randn(16, 8, device=d).to(torch.bfloat16)
    pm = torch.arange(16, dtype=torch.int32, device=d)
    probs = torch.rand(16, device=d)
    out = torch.full((16, 8), 5.0, dtype=torch.bfloat16, device=d)
    for act in (ops.MOE_ACT_SQRELU, ops.MOE_ACT_SQRELU_CLAMP):
        ops.act_with_probs_permuted(act, x, pm, torch.zeros(1, dtype=torch.int32, device=d), probs,
                                    7.0, True, out=out)
    torch.cuda.synchronize()
    assert (out == 5.0).all()                          # n_used = 0: nothing written
    eo = torch.randn(16, 8, device=d).to(torch.bfloat16)
    inv = torch.full((4, 3), -1, dtype=torch.int32, device=d)
    inv[1, 2] = 7
    uo = torch.full((4, 8), 5.0, device=d)
    ops.unpermute_ordered(eo, inv, torch.zeros(1, dtype=torch.int32, device=d), uo)
    torch.cuda.synchronize()
    assert (uo == 5.0).all()                           # valid_tokens = 0: untouched
    ops.unpermute_ordered(eo, inv, torch.full((1,), 4, dtype=torch.int32, device=d), uo)
    torch.cuda.synchronize()
    # tokens routed to no local expert get +0; token 1 gets row 7 exactly
    for t in (0, 2, 3):
        assert (bits(uo[t]).view(np.uint32) == 0).all()
    assert torch.equal(uo[1], eo[7].float())


def test_residual_fused_and_reduce_scatter_empty(cuda_device):
    d = cuda_device
    e = torch.zeros(0, 7, dtype=torch.bfloat16, device=d)
    assert ops.residual_add(e, e, e).shape == (0, 7)
    eo = torch.randn(8, 16, device=d).to(torch.bfloat16)
    inv = torch.full((3, 2), -1, dtype=torch.int32, device=d)
    sh = torch.randn(3, 16, device=d).to(torch.bfloat16)
    out = torch.full((3, 16), 5.0, dtype=torch.bfloat16, device=d)
    ops.epilogue_fused(eo, torch.rand(8, device=d), inv, torch.zeros(1, dtype=torch.int32,
                                                                      device=d), sh, sh, out=out)
    torch.cuda.synchronize()
    assert (out == 5.0).all()                          # valid_tokens = 0
    # no local expert for any token: out = residual + round(+0 + shared)
    ops.epilogue_fused(eo, torch.rand(8, device=d), inv, torch.full((1,), 3, dtype=torch.int32,
                                                                    device=d), sh, sh, out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, (sh.float() + sh.float()).to(torch.bfloat16))
    tab = ops.pointer_table([eo])
    ro = ops.ordered_reduce_scatter_v(tab, 0, torch.zeros(1, dtype=torch.int32, device=d),
                                      torch.full((1,), 8, dtype=torch.int32, device=d), 8, 16,
                                      torch.bfloat16, local_tokens=0)
    torch.cuda.synchronize()
    assert ro.shape == (0, 16)
