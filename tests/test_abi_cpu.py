"""The C-ABI library builds, loads and exports every declared symbol; host-side
argument validation rejects bad calls before anything touches a device (not gpu)."""
import os
import re

import pytest

from moe_expert_epilogue_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(_abi.SIGNATURES) <= set(names)


def test_status_strings_and_version(lib):
    assert lib.moe_abi_version() == 1
    for s in range(7):
        assert lib.moe_status_string(s).decode().startswith("MOE_")
    assert lib.moe_last_cuda_error() == 0


FAKE = 0x10000  # never dereferenced: every case below fails validation first


def _status(fn, *args):
    with pytest.raises(_abi.MoeError) as e:
        fn(*args)
    return e.value.status


def test_swiglu_validation(lib):
    f = _abi.moe_swiglu_clamped_fwd
    assert _status(f, FAKE, FAKE, FAKE, 4, 8, 16, 8, 7.0, 7, 0) == _abi.MOE_ERR_DTYPE
    assert _status(f, FAKE, FAKE, FAKE, 4, 8, 15, 8, 7.0, _abi.MOE_BF16, 0) == _abi.MOE_ERR_SHAPE
    assert _status(f, FAKE, FAKE, FAKE, -1, 8, 16, 8, 7.0, _abi.MOE_BF16, 0) == _abi.MOE_ERR_SHAPE
    for bad in (0.0, -1.0, float("nan")):
        assert _status(f, FAKE, FAKE, FAKE, 4, 8, 16, 8, bad, _abi.MOE_BF16, 0) == _abi.MOE_ERR_LIMIT
    assert _status(f, None, FAKE, FAKE, 4, 8, 16, 8, 7.0, _abi.MOE_BF16, 0) == _abi.MOE_ERR_NULL
    assert _status(f, FAKE + 1, FAKE, FAKE, 4, 8, 16, 8, 7.0, _abi.MOE_BF16, 0) == _abi.MOE_ERR_ALIGN
    assert _status(f, FAKE + 2, FAKE, FAKE, 4, 8, 16, 8, 7.0, _abi.MOE_FP32, 0) == _abi.MOE_ERR_ALIGN
    f(None, None, None, 0, 8, 16, 8, 7.0, _abi.MOE_BF16, 0)      # empty: a no-op
    b = _abi.moe_swiglu_clamped_bwd
    assert _status(b, FAKE, FAKE, FAKE, FAKE, None, 4, 8, 16, 8, 16, 7.0, 0, 0) == _abi.MOE_ERR_NULL
    assert _status(b, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 16, 8, 15, 7.0, 0, 0) == _abi.MOE_ERR_SHAPE


def test_router_weight_validation(lib):
    f = _abi.moe_router_weight_mul_fwd
    assert _status(f, FAKE, 7, FAKE, FAKE, 0, 4, 8, 0) == _abi.MOE_ERR_DTYPE
    assert _status(f, FAKE + 2, _abi.MOE_FP32, FAKE, FAKE, 0, 4, 8, 0) == _abi.MOE_ERR_ALIGN
    b = _abi.moe_router_weight_mul_bwd
    # x and grad_probs must be given together
    assert _status(b, FAKE, 0, FAKE, 0, FAKE, FAKE, None, 4, 8, 0) == _abi.MOE_ERR_NULL
    assert _status(b, FAKE, 0, None, 0, FAKE, FAKE, FAKE, 4, 8, 0) == _abi.MOE_ERR_NULL
    fx = _abi.moe_router_weight_mul_fwd_ex
    assert _status(fx, FAKE, 0, FAKE, 9, FAKE, 0, 4, 8, 0) == _abi.MOE_ERR_DTYPE
    # 16-bit probabilities need 2-byte alignment, fp32 ones 4
    assert _status(fx, FAKE, 0, FAKE + 1, _abi.MOE_BF16, FAKE, 0, 4, 8, 0) == _abi.MOE_ERR_ALIGN
    assert _status(fx, FAKE, 0, FAKE + 2, _abi.MOE_FP32, FAKE, 0, 4, 8, 0) == _abi.MOE_ERR_ALIGN
    bx = _abi.moe_router_weight_mul_bwd_ex
    assert _status(bx, FAKE, 0, FAKE, 0, FAKE, _abi.MOE_FP16, FAKE, FAKE + 1, 4, 8,
                   0) == _abi.MOE_ERR_ALIGN
    assert _status(bx, FAKE, 0, FAKE, 0, None, _abi.MOE_FP16, FAKE, FAKE, 4, 8,
                   0) == _abi.MOE_ERR_NULL


def test_permuted_and_unpermute_validation(lib):
    a = _abi.moe_act_with_probs_permuted
    assert _status(a, 9, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, 8, 1.0, 0, None, 0) == _abi.MOE_ERR_DTYPE
    for bad in (0.0, float("inf"), float("nan")):
        assert _status(a, _abi.MOE_ACT_SQRELU_CLAMP, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, 8, bad, 0,
                       None, 0) == _abi.MOE_ERR_LIMIT
    assert _status(a, 0, FAKE, FAKE, None, FAKE, FAKE, 4, 4, 8, 1.0, 0, None, 0) == _abi.MOE_ERR_NULL
    u = _abi.moe_unpermute_ordered
    assert _status(u, FAKE, 0, 4, FAKE, FAKE, FAKE, 0, 4, 8, 0, None, 0) == _abi.MOE_ERR_SHAPE
    assert _status(u, FAKE, 0, 4, FAKE, FAKE, FAKE, 0, 4, 8, 5000, None, 0) == _abi.MOE_ERR_SHAPE
    assert _status(u, FAKE, 0, 4, FAKE, FAKE + 2, FAKE, 0, 4, 8, 4, None, 0) == _abi.MOE_ERR_ALIGN


def test_reduce_scatter_validation(lib):
    f = _abi.moe_ordered_reduce_scatter_v
    ok = dict(buffers=FAKE, input_byte_offset=0, world=4, rank=1, rank_token_offset=FAKE,
              ep_tokens=FAKE, capacity_rows=100, out=FAKE, local_tokens=10, hidden=64,
              in_dt=_abi.MOE_BF16, out_dt=_abi.MOE_BF16)

    def st(**kw):
        return _status(f, *dict(ok, **kw).values())
    assert st(in_dt=5) == _abi.MOE_ERR_DTYPE
    assert st(world=0) == _abi.MOE_ERR_SHAPE and st(world=65) == _abi.MOE_ERR_SHAPE
    assert st(rank=4) == _abi.MOE_ERR_SHAPE and st(rank=-1) == _abi.MOE_ERR_SHAPE
    assert st(input_byte_offset=-16) == _abi.MOE_ERR_SHAPE
    assert st(buffers=None) == _abi.MOE_ERR_NULL and st(ep_tokens=None) == _abi.MOE_ERR_NULL
    assert st(input_byte_offset=1) == _abi.MOE_ERR_ALIGN
    assert st(buffers=FAKE + 4) == _abi.MOE_ERR_ALIGN
    assert st(out=FAKE + 2, out_dt=_abi.MOE_FP32) == _abi.MOE_ERR_ALIGN
    f(*dict(ok, local_tokens=0, buffers=None).values())          # nothing to do: a no-op


def test_ep_combine_validation(lib):
    f = _abi.moe_unpermute_reduce_scatter
    ok = dict(expert_outputs=FAKE, eo_dt=_abi.MOE_BF16, max_rows=100, inverse_maps=FAKE,
              num_local_experts=8, capacity_rows=50, ep_tokens=FAKE, world=4, rank=1,
              rank_token_offset=FAKE, partial_dt=_abi.MOE_BF16, out=FAKE, out_dt=_abi.MOE_BF16,
              local_tokens=10, hidden=64)

    def st(**kw):
        return _status(f, *dict(ok, **kw).values())
    # partial and output dtypes: the expert outputs' dtype or fp32
    assert st(partial_dt=_abi.MOE_FP16) == _abi.MOE_ERR_DTYPE
    assert st(out_dt=_abi.MOE_FP16) == _abi.MOE_ERR_DTYPE
    assert st(num_local_experts=65) == _abi.MOE_ERR_SHAPE
    assert st(num_local_experts=0) == _abi.MOE_ERR_SHAPE
    assert st(world=65) == _abi.MOE_ERR_SHAPE and st(rank=4) == _abi.MOE_ERR_SHAPE
    assert st(max_rows=2 ** 31) == _abi.MOE_ERR_SHAPE
    assert st(inverse_maps=None) == _abi.MOE_ERR_NULL
    assert st(expert_outputs=FAKE + 4) == _abi.MOE_ERR_ALIGN
    f(*dict(ok, local_tokens=0, expert_outputs=None).values())   # nothing to do: a no-op


def test_ipc_argument_checks(lib):
    import ctypes
    assert lib.moe_symm_alloc(16, None) == _abi.MOE_ERR_NULL
    assert lib.moe_ipc_export(None, ctypes.create_string_buffer(64)) == _abi.MOE_ERR_NULL
    assert lib.moe_ipc_open(None, None) == _abi.MOE_ERR_NULL
    assert lib.moe_ipc_close(None) == _abi.MOE_ERR_NULL
    assert lib.moe_symm_free(None) == _abi.MOE_OK
    with pytest.raises(ValueError):
        _abi.moe_ipc_open(b"short")


def test_residual_validation(lib):
    r = _abi.moe_residual_add
    assert _status(r, FAKE, FAKE, FAKE, FAKE, 16, 3, 0) == _abi.MOE_ERR_DTYPE
    assert _status(r, FAKE, FAKE, None, FAKE, 16, 0, 0) == _abi.MOE_ERR_NULL
    assert _status(r, FAKE, FAKE, FAKE, FAKE + 2, 16, _abi.MOE_FP32, 0) == _abi.MOE_ERR_ALIGN
    assert _status(r, FAKE, FAKE, FAKE, FAKE, -3, 0, 0) == _abi.MOE_ERR_SHAPE
    r(None, None, None, None, 0, 0, 0)                             # empty: a no-op


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "moe_expert_epilogue_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "moe_oracle" not in text, fn
