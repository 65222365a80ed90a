"""The tensor front end rejects mismatched arguments before the C ABI sees
them, and never runs on CPU tensors (not gpu).

The C ABI trusts the sizes it is given, so a wrong output shape, a wrong
dtype of a map or a count, or a non-contiguous tensor must raise in ops.py.
Tensors here are on the CPU: a call whose arguments are all consistent gets as
far as the device check and raises there -- there is no CPU fallback."""
import pytest
import torch

from moe_expert_epilogue_b200 import ops

bf, f32, i32, i64 = torch.bfloat16, torch.float32, torch.int32, torch.int64


def z(*shape, dtype=bf):
    return torch.zeros(*shape, dtype=dtype)


def _device_error(fn):
    with pytest.raises(ValueError, match="CUDA device"):
        fn()


def test_swiglu():
    x, p = z(4, 16), z(4, 1, dtype=f32)
    with pytest.raises(ValueError, match="even"):
        ops.swiglu_clamped_fwd(z(4, 15), p, 7.0)
    with pytest.raises(ValueError, match="shape"):
        ops.swiglu_clamped_fwd(x, p, 7.0, out=z(4, 16))
    with pytest.raises(TypeError, match="dtype"):
        ops.swiglu_clamped_fwd(x, p, 7.0, out=z(4, 8, dtype=f32))
    with pytest.raises(ValueError, match="elements"):
        ops.swiglu_clamped_fwd(x, z(5, dtype=f32), 7.0)
    with pytest.raises(TypeError, match="dtype"):
        ops.swiglu_clamped_fwd(x, z(4, 1), 7.0)                      # bf16 probs
    with pytest.raises(ValueError, match="unit column stride"):
        ops.swiglu_clamped_fwd(z(16, 4).t(), p, 7.0)
    with pytest.raises(ValueError, match="shape"):
        ops.swiglu_clamped_bwd(x, p, z(4, 16), 7.0)                  # grad_y [rows, 2I]
    with pytest.raises(ValueError, match="elements"):
        ops.swiglu_clamped_bwd(x, p, z(4, 8), 7.0, grad_probs=z(3, dtype=f32))
    _device_error(lambda: ops.swiglu_clamped_fwd(x, p, 7.0))
    _device_error(lambda: ops.swiglu_clamped_fwd(z(4, 40)[:, :16], p, 7.0))   # strided rows
    _device_error(lambda: ops.swiglu_clamped_bwd(x, p, z(4, 8), 7.0))


def test_router_weight():
    x, p = z(4, 8), z(4, 1, dtype=f32)
    with pytest.raises(ValueError, match="shape"):
        ops.router_weight_mul_fwd(x, p, out=z(4, 9))
    with pytest.raises(ValueError, match="contiguous"):
        ops.router_weight_mul_fwd(z(8, 4).t(), p)
    with pytest.raises(ValueError, match="elements"):
        ops.router_weight_mul_bwd(x, x, z(3, dtype=f32))
    with pytest.raises(ValueError, match="shape"):
        ops.router_weight_mul_bwd(x, z(4, 7), p)
    with pytest.raises(TypeError, match="dtype"):
        ops.router_weight_mul_bwd(x, x, p, grad_probs=z(4))          # must match probs' dtype
    _device_error(lambda: ops.router_weight_mul_fwd(x, p))
    _device_error(lambda: ops.router_weight_mul_bwd(x, None, z(4, dtype=torch.float16)))


def test_permuted_and_unpermute():
    x, pm, nu, pr = z(6, 8), z(6, dtype=i32), z(1, dtype=i32), z(10, dtype=f32)
    with pytest.raises(TypeError, match="permutation_map"):
        ops.act_with_probs_permuted(ops.MOE_ACT_SQRELU, x, z(6, dtype=i64), nu, pr)
    with pytest.raises(ValueError, match="elements"):
        ops.act_with_probs_permuted(ops.MOE_ACT_SQRELU, x, z(5, dtype=i32), nu, pr)
    with pytest.raises(ValueError, match="shape"):
        ops.act_with_probs_permuted(ops.MOE_ACT_SWIGLU, x, pm, nu, pr, out=z(6, 8))
    with pytest.raises(TypeError, match="dtype"):
        ops.act_with_probs_permuted(ops.MOE_ACT_SQRELU, z(6, 8, dtype=f32), pm, nu, pr)
    _device_error(lambda: ops.act_with_probs_permuted(ops.MOE_ACT_SWIGLU, x, pm, nu, pr))
    eo, inv, vt = z(6, 8), z(3, 4, dtype=i32), z(1, dtype=i32)
    with pytest.raises(ValueError, match="shape"):
        ops.unpermute_ordered(eo, inv, vt, z(3, 9, dtype=f32))
    with pytest.raises(TypeError, match="inverse_map"):
        ops.unpermute_ordered(eo, z(3, 4, dtype=i64), vt, z(3, 8))
    with pytest.raises(TypeError, match="valid_tokens"):
        ops.unpermute_ordered(eo, inv, z(1, dtype=i64), z(3, 8))
    _device_error(lambda: ops.unpermute_ordered(eo, inv, vt, z(3, 8, dtype=f32)))


def test_residual_bounded_fused_and_reduce_scatter():
    r = z(4, 8)
    with pytest.raises(ValueError, match="shape"):
        ops.residual_add(z(4, 9), r, r)
    with pytest.raises(TypeError, match="dtype"):
        ops.residual_add(r, z(4, 8, dtype=f32), r)
    _device_error(lambda: ops.residual_add(r, r, r, out=r))
    y, w, b = z(4, 16), z(4, dtype=f32), z(1, dtype=i64)
    with pytest.raises(TypeError, match="bound_elems"):
        ops.weighted_silu_mul_bounded(y, w, z(1, dtype=i32))
    with pytest.raises(ValueError, match="shape"):
        ops.weighted_silu_mul_bounded(y, w, b, out=z(4, 16))
    _device_error(lambda: ops.weighted_silu_mul_bounded(y, w, b))
    eo, rp, inv, vt = z(6, 8), z(6, dtype=f32), z(3, 4, dtype=i32), z(1, dtype=i32)
    sh = z(3, 8)
    with pytest.raises(ValueError, match="elements"):
        ops.epilogue_fused(eo, z(5, dtype=f32), inv, vt, sh, sh)
    with pytest.raises(ValueError, match="shape"):
        ops.epilogue_fused(eo, rp, inv, vt, z(3, 9), sh)
    with pytest.raises(TypeError, match="dtype"):
        ops.epilogue_fused(z(6, 8, dtype=f32), rp, inv, vt, sh, sh)
    _device_error(lambda: ops.epilogue_fused(eo, rp, inv, vt, sh, sh))
    tab, offs, ep = z(3, dtype=i64), z(3, dtype=i32), z(1, dtype=i32)
    with pytest.raises(ValueError, match="elements"):
        ops.ordered_reduce_scatter_v(tab, 0, z(2, dtype=i32), ep, 10, 8, bf, local_tokens=2)
    with pytest.raises(TypeError, match="buffers"):
        ops.ordered_reduce_scatter_v(z(3, dtype=i32), 0, offs, ep, 10, 8, bf, local_tokens=2)
    with pytest.raises(ValueError, match="shape"):
        ops.ordered_reduce_scatter_v(tab, 0, offs, ep, 10, 8, bf, out=z(2, 9))
    with pytest.raises(ValueError, match="local_tokens"):
        ops.ordered_reduce_scatter_v(tab, 0, offs, ep, 10, 8, bf)
    _device_error(lambda: ops.ordered_reduce_scatter_v(tab, 0, offs, ep, 10, 8, bf,
                                                       local_tokens=2))


def test_mixed_devices_are_rejected():
    class FakeCuda:
        is_cuda = True

        def __init__(self, dev):
            self.device = dev
    with pytest.raises(ValueError, match="different devices"):
        ops._cuda(FakeCuda("cuda:0"), FakeCuda("cuda:1"))


def test_ep_combine():
    tab, offs, ep = z(3, dtype=i64), z(3, dtype=i32), z(1, dtype=i32)
    with pytest.raises(ValueError, match="elements"):
        ops.unpermute_reduce_scatter(tab, bf, 10, z(2, dtype=i64), 4, 20, ep, 0, offs, 8,
                                     local_tokens=2)
    with pytest.raises(TypeError, match="inverse_maps"):
        ops.unpermute_reduce_scatter(tab, bf, 10, z(3, dtype=i32), 4, 20, ep, 0, offs, 8,
                                     local_tokens=2)
    with pytest.raises(ValueError, match="shape"):
        ops.unpermute_reduce_scatter(tab, bf, 10, tab, 4, 20, ep, 0, offs, 8, out=z(2, 9))
    _device_error(lambda: ops.unpermute_reduce_scatter(tab, bf, 10, tab, 4, 20, ep, 0, offs, 8,
                                                       local_tokens=2))
