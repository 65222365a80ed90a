"""Randomised parity sweep of every op against the CPU oracle (gpu).

Each case draws its shape, dtypes, alignment offset, leading-dimension padding
and op parameters from a seeded generator (the case index is the seed), so the
sweep reaches combinations the hand-picked tests do not -- odd widths, tiny and
ragged sizes, unaligned views that take the element-wise paths, short live
prefixes -- and every failure replays from its case index.  Pass criteria are
the ops' own: bit-exact for the router-weight multiply, the unpermute, the
residual add, the fused chain, the reduce-scatter and the EP combine; within 1 ulp of the
16-bit dtype for the SwiGLU forms and the soft-clamped squared ReLU; the
reduction tolerance for the probability gradients.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_epilogue_b200 import inputs, ops
from tests._util import assert_bits_equal, assert_sum_close, assert_within_ulp16, bits

pytestmark = pytest.mark.gpu

N_CASES = 24
DT = [torch.bfloat16, torch.float16, torch.float32]
ODT = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}
KIND = {torch.bfloat16: "bf16", torch.float16: "f16"}


def _rng(case, salt):
    return np.random.default_rng(1000 * salt + case)


def _place(t, dev, offset_elems):
    """t copied to the device at an element offset inside a larger buffer (an
    offset of 1 or 3 breaks 16-byte alignment)."""
    flat = torch.empty(t.numel() + offset_elems, dtype=t.dtype, device=dev)
    v = flat[offset_elems:].view(t.shape)
    v.copy_(t.to(dev))
    return v


def _randn(shape, sigma, seed, dtype):
    g = torch.Generator().manual_seed(int(seed))
    return (torch.randn(*shape, generator=g) * sigma).to(dtype)


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_swiglu(cuda_device, case):
    r = _rng(case, 1)
    rows, inter = int(r.integers(1, 300)), int(r.integers(1, 700))
    dt = [torch.bfloat16, torch.float16][case % 2]
    limit = float(r.choice([0.5, 3.0, 7.0, 7.3, float("inf")]))
    pad, off = int(r.integers(0, 10)), int(r.choice([0, 0, 1, 3]))
    x = _randn((rows, 2 * inter + pad), float(r.choice([1.0, 4.0])), case, dt)
    gy = _randn((rows, inter), 1.0, case + 7, dt)
    p = torch.rand(rows, 1, generator=torch.Generator().manual_seed(case))
    xd = _place(x, cuda_device, off)[:, :2 * inter]
    y = ops.swiglu_clamped_fwd(xd, p.to(cuda_device), limit)
    gx, gp = ops.swiglu_clamped_bwd(xd, p.to(cuda_device), _place(gy, cuda_device, off), limit)
    torch.cuda.synchronize()
    xb = bits(x[:, :2 * inter])
    y_ref = oracle.swiglu_clamped_fwd(xb, bits(p), limit, ODT[dt])
    gx_ref, gp_ref, gabs = oracle.swiglu_clamped_bwd(xb, bits(p), bits(gy), limit, ODT[dt])
    what = f"case {case}: rows {rows} inter {inter} pad {pad} off {off} L {limit} {dt}"
    assert_within_ulp16(bits(y), y_ref, 1, kind=KIND[dt], what="y " + what)
    assert_within_ulp16(bits(gx), gx_ref, 1, kind=KIND[dt], what="grad_x " + what)
    assert_sum_close(bits(gp).ravel(), gp_ref, gabs, 1e-5, "grad_probs " + what)


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_router_weight(cuda_device, case):
    r = _rng(case, 2)
    rows, hidden = int(r.integers(1, 400)), int(r.integers(1, 3000))
    x_dt, o_dt = DT[int(r.integers(0, 3))], DT[int(r.integers(0, 3))]
    p_dt = DT[int(r.integers(0, 3))]
    off = int(r.choice([0, 0, 1, 3]))
    x = _randn((rows, hidden), 1.0, case, x_dt)
    g = _randn((rows, hidden), 1.0, case + 1, o_dt)
    p = (torch.rand(rows, 1, generator=torch.Generator().manual_seed(case)) + 0.01).to(p_dt)
    xd, gd, pd = _place(x, cuda_device, off), _place(g, cuda_device, off), p.to(cuda_device)
    out = ops.router_weight_mul_fwd(xd, pd, o_dt)
    gx, gp = ops.router_weight_mul_bwd(gd, xd, pd)
    torch.cuda.synchronize()
    what = f"case {case}: {rows}x{hidden} x {x_dt} out {o_dt} probs {p_dt} off {off}"
    assert_bits_equal(bits(out), oracle.router_weight_fwd(bits(x), ODT[x_dt], bits(p),
                                                          ODT[o_dt], ODT[p_dt]),
                      "fwd " + what, kind=KIND.get(o_dt, "bf16"))
    gx_ref, gp_ref, gabs = oracle.router_weight_bwd(bits(g), ODT[o_dt], bits(x), ODT[x_dt],
                                                    bits(p), ODT[p_dt])
    assert_bits_equal(bits(gx), gx_ref, "grad_x " + what, kind=KIND.get(x_dt, "bf16"))
    u = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11, torch.float32: 0.0}[p_dt]
    got = gp.float().cpu().numpy().ravel().astype(np.float64)
    bound = u * np.abs(gp_ref) + 1.01e-5 * np.maximum(np.abs(gp_ref), gabs)
    assert (np.abs(got - gp_ref) <= bound).all(), "grad_probs " + what


def _routing(r, case):
    top_k = int(r.integers(1, 9))
    experts = int(r.integers(top_k, 70))
    tokens = int(r.integers(1, 200))
    align = int(r.choice([1, 4, 16, 128]))
    return inputs.routing(tokens, top_k, experts, align, seed=case)


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_permuted_activation(cuda_device, case):
    r = _rng(case, 3)
    rt = _routing(r, case)
    act, oact, tol = [(ops.MOE_ACT_SQRELU, oracle.SQRELU, 0),
                      (ops.MOE_ACT_SQRELU_CLAMP, oracle.SQRELU_CLAMP, 1),
                      (ops.MOE_ACT_SWIGLU, oracle.SWIGLU, 1)][case % 3]
    width = int(r.integers(1, 600))
    scale = float(r.choice([1.0, 7.0, 30.0]))
    zero_padding = bool(r.integers(0, 2))
    n_used = int(r.integers(0, rt.n_used + 1)) if case % 4 == 0 else rt.n_used
    x = inputs.permuted_activation_input(rt, width, swiglu=act == ops.MOE_ACT_SWIGLU,
                                         sigma=3.0, seed=case)
    canary = torch.full((rt.max_rows, width), 0x1234, dtype=torch.int16).view(torch.bfloat16)
    out = canary.to(cuda_device)
    ops.act_with_probs_permuted(act, _place(x, cuda_device, int(r.choice([0, 1]))),
                                rt.permutation_map.to(cuda_device),
                                torch.tensor([n_used], dtype=torch.int32, device=cuda_device),
                                rt.probs.to(cuda_device), scale, zero_padding, out=out)
    torch.cuda.synchronize()
    ref, err = oracle.act_with_probs_permuted(oact, bits(x), bits(canary), bits(rt.permutation_map),
                                              n_used, bits(rt.probs), width, scale, zero_padding)
    assert err == 0
    what = (f"case {case}: act {act} tokens {rt.tokens} top-{rt.top_k} of {rt.experts} align "
            f"{rt.align} width {width} n_used {n_used}/{rt.n_used}")
    if tol == 0:
        assert_bits_equal(bits(out), ref, what)
    else:
        assert_within_ulp16(bits(out), ref, tol, what=what)


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_unpermute_and_fused_chain(cuda_device, case):
    r = _rng(case, 4)
    rt = _routing(r, case)
    hidden = int(r.integers(1, 1100))
    in_dt, out_dt = DT[int(r.integers(0, 3))], DT[int(r.integers(0, 3))]
    valid = int(r.integers(0, rt.tokens + 1)) if case % 3 == 0 else rt.tokens
    eo = inputs.expert_output_input(rt, hidden, dtype=in_dt, seed=case)
    vt = torch.tensor([valid], dtype=torch.int32, device=cuda_device)
    init = torch.full((rt.tokens, hidden), 2.5, dtype=out_dt)
    out = init.to(cuda_device)
    off = int(r.choice([0, 1]))
    eod = _place(eo, cuda_device, off)
    ops.unpermute_ordered(eod, rt.inverse_map.to(cuda_device), vt, out)
    # the fused chain in the expert output's dtype
    pm = rt.permutation_map
    rp = torch.where(pm >= 0, rt.probs[pm.clamp(min=0).long()], torch.zeros(())).float()
    res = inputs.residual_inputs((rt.tokens, hidden), in_dt, seed=case)
    finit = torch.full((rt.tokens, hidden), -1.5, dtype=in_dt)
    fo = finit.to(cuda_device)
    ops.epilogue_fused(eod, rp.to(cuda_device), rt.inverse_map.to(cuda_device), vt,
                       res["shared_expert_output"].to(cuda_device),
                       res["residual"].to(cuda_device), out=fo)
    torch.cuda.synchronize()
    what = (f"case {case}: tokens {rt.tokens} top-{rt.top_k} of {rt.experts} hidden {hidden} "
            f"{in_dt}->{out_dt} valid {valid} off {off}")
    ref, err = oracle.unpermute_ordered(bits(eo), ODT[in_dt], bits(rt.inverse_map), valid,
                                        bits(init), ODT[out_dt])
    assert err == 0
    assert_bits_equal(bits(out), ref, "unpermute " + what, kind=KIND.get(out_dt, "bf16"))
    fref, ferr = oracle.epilogue_chain(bits(eo), bits(rp), bits(rt.inverse_map), valid,
                                       bits(res["shared_expert_output"]), bits(res["residual"]),
                                       bits(finit), ODT[in_dt])
    assert ferr == 0
    assert_bits_equal(bits(fo), fref, "fused " + what, kind=KIND.get(in_dt, "bf16"))


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_residual_and_bounded(cuda_device, case):
    r = _rng(case, 5)
    dt = DT[case % 3]
    n = int(r.integers(1, 100000))
    off = int(r.choice([0, 1, 3]))
    e, s, res_ = (_randn((n,), 1.0, case * 3 + k, dt) for k in range(3))
    ed, sd, rd = (_place(t, cuda_device, off) for t in (e, s, res_))
    in_place = bool(r.integers(0, 2))
    out = ops.residual_add(ed, sd, rd, out=rd if in_place else None)
    torch.cuda.synchronize()
    want = oracle.residual_add(bits(e), bits(s), bits(res_), ODT[dt])
    assert_bits_equal(bits(out), want, f"residual case {case}: n {n} {dt} off {off} "
                                       f"in place {in_place}", kind=KIND.get(dt, "bf16"))
    rows, half_n = int(r.integers(1, 300)), int(r.integers(1, 700))
    y = _randn((rows, 2 * half_n), 3.0, case, torch.bfloat16)
    w = torch.rand(rows, generator=torch.Generator().manual_seed(case))
    bound = int(r.integers(0, rows * half_n + 1))
    canary = torch.full((rows, half_n), 0x1234, dtype=torch.int16).view(torch.bfloat16)
    bo = canary.to(cuda_device)
    ops.weighted_silu_mul_bounded(_place(y, cuda_device, int(r.choice([0, 1]))),
                                  w.to(cuda_device),
                                  torch.tensor([bound], dtype=torch.int64, device=cuda_device),
                                  out=bo)
    torch.cuda.synchronize()
    bref, err = oracle.weighted_silu_mul_bounded(bits(y), bits(w), bits(canary), bound)
    assert err == 0
    assert_within_ulp16(bits(bo), bref, 1, what=f"bounded case {case}: {rows}x{half_n} "
                                                f"bound {bound}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_reduce_scatter(cuda_device, case):
    r = _rng(case, 6)
    world, tokens, hidden = int(r.integers(1, 13)), int(r.integers(0, 300)), \
        int(r.integers(1, 600))
    in_dt, out_dt = DT[int(r.integers(0, 3))], DT[int(r.integers(0, 3))]
    spare = int(r.integers(0, 4))
    rs = inputs.reduce_scatter_inputs(world, tokens, hidden, dtype=in_dt, spare_rows=spare,
                                      sigma=4.0, seed=case)
    esize = torch.empty((), dtype=in_dt).element_size()
    byte_off = esize * int(r.choice([0, 1, 8, 64]))
    cap = tokens + spare
    keep, ptrs = [], []
    for b in rs.buffers:
        raw = torch.zeros(byte_off + max(1, cap * hidden) * esize, dtype=torch.uint8,
                          device=cuda_device)
        if cap * hidden:
            raw[byte_off:byte_off + cap * hidden * esize].view(in_dt).view(cap, hidden).copy_(
                b.to(cuda_device))
        keep.append(raw)
        ptrs.append(raw.data_ptr())
    table = torch.tensor(ptrs, dtype=torch.int64, device=cuda_device)
    offs = rs.rank_token_offset.to(cuda_device)
    ep = torch.tensor([tokens], dtype=torch.int32, device=cuda_device)
    ins = [bits(b) for b in rs.buffers]
    for rank in range(world):
        init = torch.full((rs.counts[rank], hidden), -3.0, dtype=out_dt)
        out = init.to(cuda_device)
        ops.ordered_reduce_scatter_v(table, rank, offs, ep, cap, hidden, in_dt, out=out,
                                     input_byte_offset=byte_off)
        torch.cuda.synchronize()
        want, err = oracle.ordered_reduce_scatter_v(ins, ODT[in_dt], rank,
                                                    rs.rank_token_offset.numpy(), tokens,
                                                    bits(init), ODT[out_dt])
        assert err == 0
        assert_bits_equal(bits(out), want,
                          f"case {case}: world {world} rank {rank} tokens {tokens} hidden "
                          f"{hidden} {in_dt}->{out_dt} byte offset {byte_off}",
                          kind=KIND.get(out_dt, "bf16"))


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_ep_combine(cuda_device, case):
    r = _rng(case, 7)
    world = int(r.integers(1, 12))
    top_k = int(r.integers(1, 9))
    epr = int(r.integers(max(1, -(-top_k // world)), 40))
    tokens, hidden = int(r.integers(1, 200)), int(r.integers(1, 700))
    eo_dt = DT[int(r.integers(0, 3))]
    p_dt = [eo_dt, torch.float32][int(r.integers(0, 2))]
    o_dt = [eo_dt, torch.float32][int(r.integers(0, 2))]
    ec = inputs.ep_combine_inputs(world, tokens, top_k, epr, int(r.choice([1, 4, 16])), hidden,
                                  dtype=eo_dt, seed=case)
    keep = [e.to(cuda_device) for e in ec.expert_outputs] + \
        [i.to(cuda_device) for i in ec.inverse_maps]
    eo_t, inv_t = ops.pointer_table(keep[:world]), ops.pointer_table(keep[world:])
    ep = torch.tensor([tokens], dtype=torch.int32, device=cuda_device)
    offs = ec.rank_token_offset.to(cuda_device)
    eos = [bits(e) for e in ec.expert_outputs]
    invs = [bits(i) for i in ec.inverse_maps]
    for rank in range(world):
        init = torch.full((ec.counts[rank], hidden), 1.25, dtype=o_dt)
        out = init.to(cuda_device)
        ops.unpermute_reduce_scatter(eo_t, eo_dt, ec.max_rows, inv_t, epr, tokens, ep, rank, offs,
                                     hidden, out=out, partial_dtype=p_dt)
        torch.cuda.synchronize()
        want, err = oracle.unpermute_reduce_scatter(eos, ODT[eo_dt], invs, tokens, rank,
                                                    ec.rank_token_offset.numpy(), ODT[p_dt],
                                                    bits(init), ODT[o_dt])
        assert err == 0
        assert_bits_equal(bits(out), want,
                          f"case {case}: world {world} rank {rank} top-{top_k} of {world}x{epr} "
                          f"tokens {tokens} hidden {hidden} {eo_dt}/{p_dt}/{o_dt}",
                          kind=KIND.get(o_dt, "bf16"))


H16 = [torch.bfloat16, torch.float16]


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_32_byte_paths(cuda_device, case):
    """Widths that are multiples of 16 with bases offset by 0, 8 or 16 elements
    (32-byte aligned, only 16-byte aligned, 32-byte aligned again): the flat
    activation, the unpermute and fused chain, the residual add, the
    router-weight backward and the bounded SwiGLU, each against the oracle."""
    r = _rng(case, 8)
    off = int(r.choice([0, 8, 16]))
    what = f"case {case} off {off}"
    # permuted activation
    rt = _routing(r, case)
    act, oact, tol = [(ops.MOE_ACT_SQRELU, oracle.SQRELU, 0),
                      (ops.MOE_ACT_SQRELU_CLAMP, oracle.SQRELU_CLAMP, 1),
                      (ops.MOE_ACT_SWIGLU, oracle.SWIGLU, 1)][case % 3]
    width = 16 * int(r.integers(1, 100))
    zero_padding = bool(r.integers(0, 2))
    n_used = int(r.integers(0, rt.n_used + 1)) if case % 2 else rt.n_used
    x = inputs.permuted_activation_input(rt, width, swiglu=act == ops.MOE_ACT_SWIGLU, seed=case)
    canary = torch.full((rt.max_rows, width), 0x1234, dtype=torch.int16).view(torch.bfloat16)
    out = _place(canary, cuda_device, off)
    ops.act_with_probs_permuted(act, _place(x, cuda_device, off),
                                rt.permutation_map.to(cuda_device),
                                torch.tensor([n_used], dtype=torch.int32, device=cuda_device),
                                rt.probs.to(cuda_device), 7.0, zero_padding, out=out)
    torch.cuda.synchronize()
    ref, err = oracle.act_with_probs_permuted(oact, bits(x), bits(canary), bits(rt.permutation_map),
                                              n_used, bits(rt.probs), width, 7.0, zero_padding)
    assert err == 0
    w_what = f"act {act} width {width} n_used {n_used}/{rt.n_used} " + what
    if tol == 0:
        assert_bits_equal(bits(out), ref, w_what)
    else:
        assert_within_ulp16(bits(out), ref, tol, what=w_what)
    # unpermute and fused chain
    hidden = 16 * int(r.integers(1, 80))
    in_dt, out_dt = H16[int(r.integers(0, 2))], DT[int(r.integers(0, 3))]
    valid = int(r.integers(0, rt.tokens + 1))
    eo = inputs.expert_output_input(rt, hidden, dtype=in_dt, seed=case + 1)
    eod = _place(eo, cuda_device, off)
    vt = torch.tensor([valid], dtype=torch.int32, device=cuda_device)
    init = torch.full((rt.tokens, hidden), 2.5, dtype=out_dt)
    uo = _place(init, cuda_device, off)
    ops.unpermute_ordered(eod, rt.inverse_map.to(cuda_device), vt, uo)
    pm = rt.permutation_map
    rp = torch.where(pm >= 0, rt.probs[pm.clamp(min=0).long()], torch.zeros(())).float()
    res = inputs.residual_inputs((rt.tokens, hidden), in_dt, seed=case + 2)
    finit = torch.full((rt.tokens, hidden), -1.5, dtype=in_dt)
    fo = _place(finit, cuda_device, off)
    ops.epilogue_fused(eod, rp.to(cuda_device), rt.inverse_map.to(cuda_device), vt,
                       _place(res["shared_expert_output"], cuda_device, off),
                       _place(res["residual"], cuda_device, off), out=fo)
    torch.cuda.synchronize()
    u_what = f"hidden {hidden} {in_dt}->{out_dt} valid {valid}/{rt.tokens} " + what
    uref, err = oracle.unpermute_ordered(bits(eo), ODT[in_dt], bits(rt.inverse_map), valid,
                                         bits(init), ODT[out_dt])
    assert err == 0
    assert_bits_equal(bits(uo), uref, "unpermute " + u_what, kind=KIND.get(out_dt, "bf16"))
    fref, err = oracle.epilogue_chain(bits(eo), bits(rp), bits(rt.inverse_map), valid,
                                      bits(res["shared_expert_output"]), bits(res["residual"]),
                                      bits(finit), ODT[in_dt])
    assert err == 0
    assert_bits_equal(bits(fo), fref, "fused " + u_what, kind=KIND.get(in_dt, "bf16"))
    # residual add, possibly in place
    dt = H16[case % 2]
    n = int(r.integers(1, 200000))
    e, s, rr = (_randn((n,), 1.0, case * 3 + k, dt) for k in range(3))
    ed, sd, rd = (_place(t, cuda_device, off) for t in (e, s, rr))
    in_place = bool(r.integers(0, 2))
    ro = ops.residual_add(ed, sd, rd, out=rd if in_place else None)
    torch.cuda.synchronize()
    assert_bits_equal(bits(ro), oracle.residual_add(bits(e), bits(s), bits(rr), ODT[dt]),
                      f"residual n {n} in place {in_place} " + what, kind=KIND[dt])
    # router-weight backward with x saved
    rows, rh = int(r.integers(1, 300)), 16 * int(r.integers(1, 500))
    g_dt, x_dt = H16[int(r.integers(0, 2))], H16[int(r.integers(0, 2))]
    xw = _randn((rows, rh), 1.0, case + 3, x_dt)
    gw = _randn((rows, rh), 1.0, case + 4, g_dt)
    pw = torch.rand(rows, 1, generator=torch.Generator().manual_seed(case)) + 0.01
    gx, gp = ops.router_weight_mul_bwd(_place(gw, cuda_device, off), _place(xw, cuda_device, off),
                                       pw.to(cuda_device))
    torch.cuda.synchronize()
    gx_ref, gp_ref, gabs = oracle.router_weight_bwd(bits(gw), ODT[g_dt], bits(xw), ODT[x_dt],
                                                    bits(pw))
    rw_what = f"router bwd {rows}x{rh} g {g_dt} x {x_dt} " + what
    assert_bits_equal(bits(gx), gx_ref, "grad_x " + rw_what, kind=KIND[x_dt])
    assert_sum_close(bits(gp).ravel(), gp_ref, gabs, 1e-5, "grad_probs " + rw_what)
    # bounded weighted SwiGLU
    brows, half_n = int(r.integers(1, 300)), 16 * int(r.integers(1, 60))
    y = _randn((brows, 2 * half_n), 3.0, case + 5, torch.bfloat16)
    wb = torch.rand(brows, generator=torch.Generator().manual_seed(case + 6))
    bound = int(r.integers(0, brows * half_n + 1))
    bcan = torch.full((brows, half_n), 0x1234, dtype=torch.int16).view(torch.bfloat16)
    bo = _place(bcan, cuda_device, off)
    ops.weighted_silu_mul_bounded(_place(y, cuda_device, off), wb.to(cuda_device),
                                  torch.tensor([bound], dtype=torch.int64, device=cuda_device),
                                  out=bo)
    torch.cuda.synchronize()
    bref, err = oracle.weighted_silu_mul_bounded(bits(y), bits(wb), bits(bcan), bound)
    assert err == 0
    assert_within_ulp16(bits(bo), bref, 1, what=f"bounded {brows}x{half_n} bound {bound} " + what)
