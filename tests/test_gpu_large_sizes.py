"""Maximum sizes (gpu): every kernel on tensors of more than 2^31 elements.

Each case puts an element index, a row offset or a source offset past 2^31,
so a 32-bit product anywhere in a kernel's addressing would show as wrong
values there.  Outputs are checked against the CPU oracle on sampled rows:
the first ones, those on both sides of the 2^31-element boundary, the last
ones (with a ragged tail where the op has one) and a random draw.  Inputs are
drawn on the device (seeded) and freed after each case; a GPU with less free
memory than a case needs skips it.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_epilogue_b200 import inputs, ops
from tests._util import assert_bits_equal, assert_sum_close, assert_within_ulp16, bits

pytestmark = pytest.mark.gpu

B31 = 2 ** 31


@pytest.fixture
def big_device(cuda_device):
    yield cuda_device
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _need(dev, gib):
    free, _ = torch.cuda.mem_get_info(dev)
    if free < gib * 2 ** 30:
        pytest.skip(f"needs {gib} GiB of free device memory")


def _randn(shape, dev, seed, sigma=1.0, dtype=torch.bfloat16):
    g = torch.Generator(device=dev).manual_seed(seed)
    out = torch.empty(shape, dtype=dtype, device=dev)
    flat = out.view(-1)
    step = 1 << 28                                   # keep the fp32 temporary small
    for i in range(0, flat.numel(), step):
        n = min(step, flat.numel() - i)
        flat[i:i + n] = (torch.randn(n, generator=g, device=dev) * sigma).to(dtype)
    return out


def _sample_rows(rows, row_elems, seed, n_random=200):
    """Rows 0..3, the rows around element 2^31, the last 4 rows, and a draw."""
    b = B31 // row_elems
    idx = [0, 1, 2, 3, b - 1, b, b + 1, rows - 4, rows - 3, rows - 2, rows - 1]
    idx += list(np.random.default_rng(seed).integers(0, rows, n_random))
    return np.unique(np.clip(np.array(idx), 0, rows - 1))


def test_residual_add_past_2_31_elements(big_device):
    n = B31 + 8 * 1000 + 3                                # vector body + ragged tail
    _need(big_device, 18)
    e, s, r = (_randn((n,), big_device, 10 + k) for k in range(3))
    out = ops.residual_add(e, s, r)
    torch.cuda.synchronize()
    idx = np.unique(np.concatenate([
        np.arange(16), np.arange(B31 - 16, B31 + 16), np.arange(n - 40, n),
        np.random.default_rng(1).integers(0, n, 2000)]))
    ti = torch.from_numpy(idx).to(big_device)
    want = oracle.residual_add(bits(e[ti]), bits(s[ti]), bits(r[ti]), oracle.BF16)
    assert_bits_equal(bits(out[ti]), want, "residual add")


def test_router_weight_past_2_31_elements(big_device):
    rows, hidden = 300000, 7168                           # 2.15e9 elements
    _need(big_device, 20)
    x = _randn((rows, hidden), big_device, 20)
    g = _randn((rows, hidden), big_device, 21)
    p = torch.rand(rows, 1, generator=torch.Generator(device=big_device).manual_seed(22),
                   device=big_device) * 0.99 + 0.01
    out = ops.router_weight_mul_fwd(x, p, torch.bfloat16)
    gx, gp = ops.router_weight_mul_bwd(g, x, p)
    torch.cuda.synchronize()
    idx = torch.from_numpy(_sample_rows(rows, hidden, 2)).to(big_device)
    xb, pb, gb = bits(x[idx]), bits(p[idx]), bits(g[idx])
    assert_bits_equal(bits(out[idx]), oracle.router_weight_fwd(xb, oracle.BF16, pb, oracle.BF16),
                      "fwd")
    gx_ref, gp_ref, gabs = oracle.router_weight_bwd(gb, oracle.BF16, xb, oracle.BF16, pb)
    assert_bits_equal(bits(gx[idx]), gx_ref, "grad_x")
    assert_sum_close(bits(gp[idx]).ravel(), gp_ref, gabs, 1e-5, "grad_probs")


def test_swiglu_fwd_bwd_past_2_31_elements(big_device):
    rows, inter = 524300, 2048                            # x: 2.15e9 elements
    _need(big_device, 16)
    x = _randn((rows, 2 * inter), big_device, 30, sigma=3.0)
    gy = _randn((rows, inter), big_device, 31)
    p = torch.rand(rows, 1, generator=torch.Generator(device=big_device).manual_seed(32),
                   device=big_device)
    y = ops.swiglu_clamped_fwd(x, p, 10.0)
    gx, gp = ops.swiglu_clamped_bwd(x, p, gy, 10.0)
    torch.cuda.synchronize()
    idx = torch.from_numpy(_sample_rows(rows, 2 * inter, 3)).to(big_device)
    xb, pb, gb = bits(x[idx]), bits(p[idx]), bits(gy[idx])
    assert_within_ulp16(bits(y[idx]), oracle.swiglu_clamped_fwd(xb, pb, 10.0), 1, what="fwd")
    gx_ref, gp_ref, gabs = oracle.swiglu_clamped_bwd(xb, pb, gb, 10.0)
    assert_within_ulp16(bits(gx[idx]), gx_ref, 1, what="grad_x")
    assert_sum_close(bits(gp[idx]).ravel(), gp_ref, gabs, 1e-5, "grad_probs")


def _big_routing(dev):
    # 65600 tokens x top-8 of 64 experts, padded to 128: max_rows 532992
    return inputs.routing(65600, 8, 64, 128, seed=40, device=dev)


def _compact_rows(rt, eo, tok):
    """The expert-output rows the sampled tokens read, gathered, with the
    tokens' inverse-map rows renumbered into the gathered block (the sum order
    depends on the expert index only, so renumbering keeps every bit)."""
    inv = rt.inverse_map[tok].cpu().numpy()
    used = np.unique(inv[inv >= 0])
    remap = np.full(rt.max_rows, -1, np.int64)
    remap[used] = np.arange(used.size)
    inv_c = np.where(inv >= 0, remap[np.maximum(inv, 0)], -1).astype(np.int32)
    rows = torch.from_numpy(used).to(eo.device)
    return used, inv_c, rows


def test_unpermute_and_fused_chain_past_2_31_elements(big_device):
    _need(big_device, 24)
    rt = _big_routing(big_device)
    H = 4096
    eo = inputs.expert_output_input(rt, H, seed=41, device=big_device)   # 2.18e9 elements
    vt = torch.tensor([rt.tokens], dtype=torch.int32, device=big_device)
    out = torch.empty(rt.tokens, H, dtype=torch.float32, device=big_device)
    ops.unpermute_ordered(eo, rt.inverse_map, vt, out)
    pm = rt.permutation_map
    rp = torch.where(pm >= 0, rt.probs[pm.clamp(min=0).long()],
                     torch.zeros((), device=big_device)).float()
    res = inputs.residual_inputs((rt.tokens, H), torch.bfloat16, seed=42, device=big_device)
    fo = ops.epilogue_fused(eo, rp, rt.inverse_map, vt, res["shared_expert_output"],
                            res["residual"])
    torch.cuda.synchronize()
    # tokens whose rows lie past element 2^31 (the last experts' blocks) and a draw
    inv = rt.inverse_map.cpu().numpy()
    far = np.nonzero((inv.max(axis=1).astype(np.int64) * H) >= B31)[0]
    tok = np.unique(np.concatenate([far[:40], far[-40:], [0, rt.tokens - 1],
                                    np.random.default_rng(4).integers(0, rt.tokens, 100)]))
    assert far.size > 0
    used, inv_c, rows = _compact_rows(rt, eo, tok)
    eo_c = bits(eo[rows])
    ref, err = oracle.unpermute_ordered(eo_c, oracle.BF16, inv_c, tok.size,
                                        np.zeros((tok.size, H), np.float32), oracle.F32)
    assert err == 0
    tt = torch.from_numpy(tok).to(big_device)
    assert np.array_equal(bits(out[tt]).view(np.uint32), ref.view(np.uint32)), "unpermute"
    fref, ferr = oracle.epilogue_chain(eo_c, bits(rp[rows]), inv_c, tok.size,
                                       bits(res["shared_expert_output"][tt]),
                                       bits(res["residual"][tt]),
                                       np.zeros((tok.size, H), np.uint16), oracle.BF16)
    assert ferr == 0
    assert_bits_equal(bits(fo[tt]), fref, "fused chain")


def test_permuted_swiglu_past_2_31_elements(big_device):
    _need(big_device, 24)
    rt = _big_routing(big_device)
    W = 2048                                              # input 532992 x 4096 = 2.18e9
    x = inputs.permuted_activation_input(rt, W, swiglu=True, seed=43, device=big_device)
    nu = torch.tensor([rt.n_used], dtype=torch.int32, device=big_device)
    out = torch.zeros(rt.max_rows, W, dtype=torch.bfloat16, device=big_device)
    ops.act_with_probs_permuted(ops.MOE_ACT_SWIGLU, x, rt.permutation_map, nu, rt.probs, 1.0,
                                True, out=out)
    torch.cuda.synchronize()
    live = rt.n_used
    idx = _sample_rows(live, 2 * W, 5)
    ti = torch.from_numpy(idx).to(big_device)
    ref, err = oracle.act_with_probs_permuted(oracle.SWIGLU, bits(x[ti]),
                                              np.zeros((idx.size, W), np.uint16),
                                              bits(rt.permutation_map[ti]), idx.size,
                                              bits(rt.probs), W, 1.0, True)
    assert err == 0
    assert_within_ulp16(bits(out[ti]), ref, 1, what="permuted swiglu")


def test_bounded_swiglu_past_2_31_elements(big_device):
    rows, half_n = 524300, 2048                           # y: 2.15e9 elements
    _need(big_device, 12)
    y = _randn((rows, 2 * half_n), big_device, 50, sigma=3.0)
    w = torch.rand(rows, generator=torch.Generator(device=big_device).manual_seed(51),
                   device=big_device)
    bound = (rows - 2) * half_n + 5
    out = torch.zeros(rows, half_n, dtype=torch.bfloat16, device=big_device)
    ops.weighted_silu_mul_bounded(y, w, torch.tensor([bound], dtype=torch.int64,
                                                     device=big_device), out=out)
    torch.cuda.synchronize()
    idx = _sample_rows(rows - 2, 2 * half_n, 6)
    ti = torch.from_numpy(idx).to(big_device)
    ref, _ = oracle.weighted_silu_mul_bounded(bits(y[ti]), bits(w[ti]),
                                              np.zeros((idx.size, half_n), np.uint16),
                                              idx.size * half_n)
    assert_within_ulp16(bits(out[ti]), ref, 1, what="bounded")
    tail = bits(out[rows - 2:])
    assert (tail[0, 5:] == 0).all() and (tail[1] == 0).all()


def test_reduce_scatter_past_2_31_elements(big_device):
    """2 ranks' blocks of 600000 x 4096 (2.46e9 elements each); rank 1's rows
    start past element 2^31 of every block."""
    _need(big_device, 24)
    T, H = 600000, 4096
    blocks = [_randn((T, H), big_device, 60 + q) for q in range(2)]
    offs = torch.tensor([0, 530000], dtype=torch.int32, device=big_device)
    ep = torch.tensor([T], dtype=torch.int32, device=big_device)
    table = ops.pointer_table(blocks)
    out = ops.ordered_reduce_scatter_v(table, 1, offs, ep, T, H, torch.bfloat16,
                                       local_tokens=T - 530000)
    torch.cuda.synchronize()
    idx = np.unique(np.concatenate([[0, 1, T - 530000 - 1],
                                    np.random.default_rng(7).integers(0, T - 530000, 100)]))
    src = torch.from_numpy(idx + 530000).to(big_device)
    ins = [bits(b[src]) for b in blocks]
    ref, err = oracle.ordered_reduce_scatter_v(ins, oracle.BF16, 0, [0, 0], idx.size,
                                               np.zeros((idx.size, H), np.uint16), oracle.BF16)
    assert err == 0
    assert_bits_equal(bits(out[torch.from_numpy(idx).to(big_device)]), ref, "reduce-scatter")
