"""B200 (sm_100a) MoE expert-epilogue library.

Seven memory-bound ops behind a C ABI (include/moe_epilogue.h), implemented as
hand-written CUDA kernels in csrc/ and built into libmoe_epilogue.so:

    moe_swiglu_clamped_fwd / moe_swiglu_clamped_bwd
    moe_router_weight_mul_fwd / moe_router_weight_mul_bwd
    moe_act_with_probs_permuted
    moe_unpermute_ordered
    moe_residual_add
    moe_weighted_silu_mul_bounded
    moe_epilogue_fused

``_abi`` is the ctypes binding with the C names and argument order; ``ops``
is a tensor-level front end that allocates outputs with torch.  ``inputs``
draws the seeded synthetic workloads.
"""
from . import _abi  # noqa: F401
from ._abi import (MOE_ACT_SQRELU, MOE_ACT_SQRELU_CLAMP, MOE_ACT_SWIGLU,  # noqa: F401
                   MOE_BF16, MOE_FP16, MOE_FP32, MoeError, moe_act_with_probs_permuted,
                   moe_residual_add, moe_router_weight_mul_bwd, moe_router_weight_mul_fwd,
                   moe_swiglu_clamped_bwd, moe_swiglu_clamped_fwd, moe_unpermute_ordered,
                   moe_weighted_silu_mul_bounded, moe_epilogue_fused)
