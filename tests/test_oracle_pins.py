"""Pins for the CPU oracle (not gpu).

Each test checks the oracle against something other than itself: a library
routine (torch / numpy conversions, torch autograd, torch.clamp / F.silu /
torch.tanh in float64 or fp32), a closed form, float64 finite differences, an
exact-arithmetic construction, or a stored special-value fixture under
tests/golden/.  Together they are chosen so that a dropped term, a wrong sign,
a swapped gate/up half, a wrong mask boundary or a wrong rounding step fails at
least one of them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from moe_expert_epilogue_b200 import inputs
from tests._util import (assert_bits_equal, assert_sum_close, assert_within_ulp16, bits,
                         from_bits, ulp_diff16)

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- dtypes

def _probe_floats(n=20000, seed=0):
    rng = np.random.default_rng(seed)
    mant = rng.integers(0, 1 << 23, n, dtype=np.uint32)
    exp = rng.integers(0, 255, n, dtype=np.uint32)
    sign = rng.integers(0, 2, n, dtype=np.uint32) << 31
    x = (sign | (exp << 23) | mant).view(np.float32)
    # exact bf16 ties (lower 16 bits == 0x8000) with odd and even kept parts
    ties = (rng.integers(0, 1 << 16, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    specials = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 3.3895314e38, -3.3895314e38,
                         65504.0, 65519.996, 65520.0, 6.0e-8, 2.9802322e-08, 2.9802326e-08,
                         5.9604645e-08, 1e-45, 1.17549435e-38], np.float32)
    return np.concatenate([x, ties, specials])


def test_bf16_rounding_matches_torch():
    x = _probe_floats()
    got = oracle.bf16_from_f32(x)
    want = bits(torch.from_numpy(x).to(torch.bfloat16))
    assert_bits_equal(got, want, "bf16 RNE")
    back = oracle.f32_from_bf16(got)
    assert_bits_equal(back, torch.from_numpy(got.view(np.int16)).view(torch.bfloat16)
                      .float().numpy(), "bf16 widen")


def test_f16_rounding_matches_numpy():
    x = _probe_floats(seed=1)
    # binary16 ties and the subnormal range, where numpy rounds to nearest even
    rng = np.random.default_rng(2)
    sub = (rng.random(5000) * 2.0 ** -14).astype(np.float32)
    tie = (np.arange(1, 2000, dtype=np.float32) * 2.0 ** -25).astype(np.float32)
    x = np.concatenate([x, sub, -sub, tie])
    with np.errstate(over="ignore", invalid="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    got = oracle.f16_from_f32(x)
    assert_bits_equal(got, want, "f16 RNE", kind="f16")
    back = oracle.f32_from_f16(got)
    assert_bits_equal(back, got.view(np.float16).astype(np.float32), "f16 widen")


# ------------------------------------------------------ clamped SwiGLU fwd

def _swiglu_ref64(x_bits, probs, limit):
    """Library chain in float64: F.silu(torch.clamp(g, max=L)) *
    torch.clamp(u, -L, L) * p, rounded once to bf16 by torch."""
    x = from_bits(x_bits, torch.bfloat16).double()
    inter = x.shape[1] // 2
    g, u = x[:, :inter], x[:, inter:]
    p = torch.from_numpy(np.asarray(probs, np.float32)).double().reshape(-1, 1)
    y = F.silu(torch.clamp(g, max=limit)) * torch.clamp(u, -limit, limit) * p
    return bits(y.to(torch.bfloat16))


@pytest.mark.parametrize("limit", [7.0, 7.3, 10.0, float("inf")])
def test_swiglu_fwd_vs_float64_library_chain(limit):
    d = inputs.swiglu_inputs(64, 96, sigma=4.0, limit=limit if limit == 7.0 else None,
                             plant_ties=(limit == 7.0), seed=3)
    xb, p = bits(d["x"]), bits(d["probs"])
    got = oracle.swiglu_clamped_fwd(xb, p, limit)
    dist = assert_within_ulp16(got, _swiglu_ref64(xb, p, limit), 1, what="fwd")
    assert (dist == 0).mean() > 0.99


def test_swiglu_fwd_plain_swiglu_when_unclamped_and_unweighted():
    # limit = inf and probs = 1 reduce the op to plain SwiGLU silu(g) * u,
    # evaluated by torch in fp32.
    d = inputs.swiglu_inputs(128, 64, sigma=3.0, seed=4)
    xb = bits(d["x"])
    ones = np.ones(128, np.float32)
    got = oracle.swiglu_clamped_fwd(xb, ones, float("inf"))
    x = d["x"].float()
    want = bits((F.silu(x[:, :64]) * x[:, 64:]).to(torch.bfloat16))
    dist = assert_within_ulp16(got, want, 1, what="plain swiglu")
    assert (dist == 0).mean() > 0.99


def test_swiglu_fwd_closed_forms():
    L = 7.0
    vals = [  # gate, up, prob, exact y (float64 closed form)
        (0.0, 3.0, 0.5, 0.0),                                  # silu(0) = 0
        (2.0, 0.0, 0.5, 0.0),                                  # up = 0
        (1.0, 1.0, 0.0, 0.0),                                  # prob = 0
        (9.0, 1.0, 1.0, L / (1 + math.exp(-L))),               # gate saturates at L
        (64.0, -50.0, 0.25, -L * L / (1 + math.exp(-L)) * 0.25),  # both clamp
        (-3.0, 12.0, 1.0, -3.0 / (1 + math.exp(3.0)) * L),     # up clamps at +L only
    ]
    x = torch.tensor([[g, u] for g, u, _, _ in vals], dtype=torch.bfloat16)
    p = np.array([v[2] for v in vals], np.float32)
    got = oracle.swiglu_clamped_fwd(bits(x), p, L)[:, 0]
    want = bits(torch.tensor([v[3] for v in vals], dtype=torch.float64).to(torch.bfloat16))
    assert_within_ulp16(got, want, 1, what="closed forms")
    assert got[0] == 0 and got[1] in (0, 0x8000) and got[2] in (0, 0x8000)


def test_swiglu_fwd_nan_propagates_like_torch_clamp():
    x = torch.tensor([[float("nan"), 1.0], [1.0, float("nan")]], dtype=torch.bfloat16)
    y = oracle.swiglu_clamped_fwd(bits(x), np.ones(2, np.float32), 7.0)
    assert ((y & 0x7F80) == 0x7F80).all() and ((y & 0x7F) != 0).all()


def test_swiglu_golden_special_values():
    """Fixture of hand-derived values (tests/golden/swiglu_special_values.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "swiglu_special_values.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    for gate, up, prob, limit, want in rows:
        x = torch.tensor([[float(gate), float(up)]], dtype=torch.bfloat16)
        assert float(x[0, 0]) == float(gate) and float(x[0, 1]) == float(up)
        y = oracle.swiglu_clamped_fwd(bits(x), np.array([float(prob)], np.float32),
                                      float(limit))
        got = float(torch.from_numpy(y.view(np.int16)).view(torch.bfloat16)[0, 0])
        assert got == float(want), (gate, up, prob, limit, got, want)


# ------------------------------------------------------ clamped SwiGLU bwd

def _autograd64(x_bits, probs, grad_y_bits, limit):
    x = from_bits(x_bits, torch.bfloat16).double().requires_grad_(True)
    inter = x.shape[1] // 2
    p = torch.from_numpy(np.asarray(probs, np.float32)).double().reshape(-1, 1)
    p.requires_grad_(True)
    dy = from_bits(grad_y_bits, torch.bfloat16).double()
    y = F.silu(torch.clamp(x[:, :inter], max=limit)) * torch.clamp(x[:, inter:], -limit,
                                                                   limit) * p
    y.backward(dy)
    return x.grad, p.grad.reshape(-1)


@pytest.mark.parametrize("limit", [7.0, float("inf")])
def test_swiglu_bwd_vs_float64_autograd(limit):
    d = inputs.swiglu_inputs(48, 80, sigma=3.0, limit=limit if limit != float("inf") else None,
                             plant_ties=(limit != float("inf")), seed=5)
    xb, p, gyb = bits(d["x"]), bits(d["probs"]), bits(d["grad_y"])
    gx, gp, gabs = oracle.swiglu_clamped_bwd(xb, p, gyb, limit)
    ref_gx, ref_gp = _autograd64(xb, p, gyb, limit)
    dist = assert_within_ulp16(gx, bits(ref_gx.to(torch.bfloat16)), 1, what="grad_x")
    assert (dist == 0).mean() > 0.99
    assert_sum_close(gp, ref_gp.numpy(), gabs, 1e-6, "grad_probs")


def test_swiglu_bwd_inclusive_masks_at_planted_ties():
    L = 7.0
    above = float(torch.tensor(L, dtype=torch.bfloat16).view(torch.int16).add(1)
                  .view(torch.bfloat16))
    g = [L, above, 1.0, 1.0, 1.0, 1.0]
    u = [2.0, 2.0, L, -L, above, -above]
    x = torch.tensor([g + u], dtype=torch.bfloat16)
    gy = torch.ones(1, 6, dtype=torch.bfloat16)
    gx, _, _ = oracle.swiglu_clamped_bwd(bits(x), np.ones(1, np.float32), bits(gy), L)
    gate_grad, up_grad = gx[0, :6], gx[0, 6:]
    assert gate_grad[0] != 0          # g == L: inside the inclusive range
    assert gate_grad[1] == 0          # g just above L: clamped, gradient 0
    assert up_grad[2] != 0 and up_grad[3] != 0    # u == +-L: inside
    assert up_grad[4] == 0 and up_grad[5] == 0    # just outside
    ref_gx, _ = _autograd64(bits(x), np.ones(1, np.float32), bits(gy), L)
    assert_within_ulp16(gx, bits(ref_gx.to(torch.bfloat16)), 1, what="ties vs autograd")


def test_swiglu_bwd_vs_float64_finite_differences():
    """Tiny inputs (R=3, I=5) away from the clamp kinks: the oracle's bf16
    gradients agree with central differences of the float64 twin of the
    forward, and the twin agrees with the fp32 forward."""
    rng = np.random.default_rng(6)
    L = 4.0
    R, I = 3, 5
    g = rng.uniform(-6, 3.5, (R, I))
    u = rng.uniform(-3.5, 3.5, (R, I))
    g[0, 0], u[1, 1] = 5.5, -5.0                       # beyond the limit: zero slope
    x = torch.tensor(np.concatenate([g, u], 1), dtype=torch.bfloat16)
    xb = bits(x)
    g = x[:, :I].double().numpy()
    u = x[:, I:].double().numpy()
    p = np.array([0.3, 0.9, 0.55], np.float32)
    dy = torch.tensor(rng.standard_normal((R, I)), dtype=torch.bfloat16)
    dyd = dy.double().numpy()
    pp = np.repeat(p.astype(np.float64)[:, None], I, 1)

    y32 = oracle.swiglu_clamped_fwd(xb, p, L)
    y64 = oracle.swiglu_clamped_fwd_f64(g, u, pp, L).reshape(R, I)
    assert_within_ulp16(y32, bits(torch.from_numpy(y64).to(torch.bfloat16)), 1, what="twin")

    h = 1e-6
    f = lambda gg, uu, ppp: oracle.swiglu_clamped_fwd_f64(gg, uu, ppp, L).reshape(R, I)
    d_g = (f(g + h, u, pp) - f(g - h, u, pp)) / (2 * h) * dyd
    d_u = (f(g, u + h, pp) - f(g, u - h, pp)) / (2 * h) * dyd
    d_p = ((f(g, u, pp + h) - f(g, u, pp - h)) / (2 * h) * dyd).sum(1)
    gx, gp, gabs = oracle.swiglu_clamped_bwd(xb, p, bits(dy), L)
    fd = np.concatenate([d_g, d_u], 1)
    assert_within_ulp16(gx, bits(torch.from_numpy(fd).to(torch.bfloat16)), 1, what="FD grad_x")
    assert gx[0, 0] == 0 and gx[1, I + 1] == 0
    np.testing.assert_allclose(gp, d_p, rtol=1e-5, atol=1e-7)


# ------------------------------------------------------ router weight

DT = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}


@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32, torch.float16])
def test_router_weight_fwd_bitwise_vs_torch(x_dtype, out_dtype):
    d = inputs.router_weight_inputs(33, 70, seed=7)
    x = d["x"].to(x_dtype)
    want = (x.float() * d["probs"].float()).to(out_dtype)      # the documented definition
    got = oracle.router_weight_fwd(bits(x), DT[x_dtype], bits(d["probs"]), DT[out_dtype])
    assert_bits_equal(got, bits(want), "rw fwd")


@pytest.mark.parametrize("g_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("save_x", [True, False])
def test_router_weight_bwd_vs_torch_autograd(g_dtype, save_x):
    d = inputs.router_weight_inputs(40, 300, out_dtype=g_dtype, seed=8)
    x = d["x"].clone().requires_grad_(True)
    p = d["probs"].clone().requires_grad_(True)
    out = (x.float() * p.float()).to(g_dtype)                   # autograd's fp32 chain
    out.backward(d["grad_out"])
    gx, gp, gabs = oracle.router_weight_bwd(bits(d["grad_out"]), DT[g_dtype],
                                            bits(d["x"]) if save_x else None, oracle.BF16,
                                            bits(d["probs"]))
    assert_bits_equal(gx, bits(x.grad), "grad_x")
    if save_x:
        assert_sum_close(gp, p.grad.reshape(-1).double().numpy(), gabs, 1e-5, "grad_probs")
    else:
        assert gp is None


# ------------------------------------------------------ permuted activation

def _tiny_routing():
    return inputs.routing(tokens=12, top_k=2, experts=4, align=4, seed=9)


def _loop_ref(act, x, rt, width, scale):
    """Per live row, the library chain in torch (bf16 tensor ops round each op
    to bf16; fp32 tensors round nothing until .to(bf16))."""
    out = {}
    for r in range(rt.n_used):
        m = int(rt.permutation_map[r])
        if m < 0:
            continue
        p = rt.probs[m].float()
        row = x[r]
        if act == oracle.SQRELU:
            rl = torch.relu(row)                  # bf16
            sq = rl * rl                          # bf16 square: one rounding
            out[r] = (sq.float() * p).to(torch.bfloat16)
        elif act == oracle.SQRELU_CLAMP:
            z = scale * torch.tanh(row.float() / scale)
            out[r] = (torch.relu(z).square() * p).to(torch.bfloat16)
        else:
            gte, up = row[:width].float(), row[width:].float()
            out[r] = (F.silu(gte) * up * p).to(torch.bfloat16)
    return out


@pytest.mark.parametrize("act", [oracle.SQRELU, oracle.SQRELU_CLAMP, oracle.SWIGLU])
@pytest.mark.parametrize("zero_padding", [False, True])
def test_act_permuted_brute_force(act, zero_padding):
    rt = _tiny_routing()
    width = 24
    scale = 7.0
    x = inputs.permuted_activation_input(rt, width, swiglu=(act == oracle.SWIGLU), seed=10)
    canary = np.full((rt.max_rows, width), 0x1234, np.uint16)
    got, err = oracle.act_with_probs_permuted(act, bits(x), canary, bits(rt.permutation_map),
                                              rt.n_used, bits(rt.probs), width, scale,
                                              zero_padding)
    assert err == 0
    ref = _loop_ref(act, x, rt, width, scale)
    pm = rt.permutation_map.numpy()
    for r in range(rt.max_rows):
        if r in ref:
            tol = 0 if act == oracle.SQRELU else 1
            assert_within_ulp16(got[r], bits(ref[r]), tol, what=f"row {r}")
        elif r < rt.n_used and pm[r] < 0 and zero_padding:
            assert (got[r] == 0).all()
        else:
            assert (got[r] == 0x1234).all(), f"row {r} touched"


def test_sqrelu_rounding_witness():
    """Without CLAMP the square is rounded to bf16 before the probability
    multiply; with CLAMP (and a scale so large that s*tanh(x/s) == x) there is
    one rounding only.  Pick x, p where the two differ and check each branch."""
    xs = torch.arange(1, 400, dtype=torch.float32).mul(0.0371).to(torch.bfloat16)
    p = torch.tensor(0.7071, dtype=torch.float32)
    double = ((xs * xs).float() * p).to(torch.bfloat16)
    single = ((xs.float() * xs.float()) * p).to(torch.bfloat16)
    witness = torch.nonzero(double != single).flatten()
    assert witness.numel() > 0
    i = int(witness[0])
    rt = inputs.Routing(1, 1, 1, 1, 1, 1, torch.tensor([0], dtype=torch.int32),
                        torch.tensor([[0]], dtype=torch.int32), p.reshape(1),
                        torch.tensor([1]))
    x = xs[i].reshape(1, 1)
    big = float(2.0 ** 100)
    o1, _ = oracle.act_with_probs_permuted(oracle.SQRELU, bits(x), np.zeros((1, 1), np.uint16),
                                           np.array([0], np.int32), 1, bits(rt.probs), 1)
    o2, _ = oracle.act_with_probs_permuted(oracle.SQRELU_CLAMP, bits(x),
                                           np.zeros((1, 1), np.uint16),
                                           np.array([0], np.int32), 1, bits(rt.probs), 1, big)
    assert o1[0, 0] == bits(double[i].reshape(1))[0]
    assert o2[0, 0] == bits(single[i].reshape(1))[0]


def test_act_permuted_reports_bad_metadata():
    rt = _tiny_routing()
    x = inputs.permuted_activation_input(rt, 8, swiglu=False, seed=11)
    out0 = np.zeros((rt.max_rows, 8), np.uint16)
    _, err = oracle.act_with_probs_permuted(oracle.SQRELU, bits(x), out0,
                                            bits(rt.permutation_map), rt.max_rows + 5,
                                            bits(rt.probs), 8)
    assert err & oracle.ERR_COUNT
    pm = bits(rt.permutation_map).copy()
    live = np.flatnonzero(pm >= 0)
    pm[live[0]] = 10 ** 6
    out, err = oracle.act_with_probs_permuted(oracle.SQRELU, bits(x), out0, pm, rt.n_used,
                                              bits(rt.probs), 8)
    assert err == oracle.ERR_MAP and (out[live[0]] == 0).all()


# ------------------------------------------------------ unpermute

def test_unpermute_exact_integer_sums():
    """Small-integer expert outputs: every fp32 partial sum is exact, so the
    result is the integer sum, computed here with int64 arithmetic."""
    rt = inputs.routing(tokens=20, top_k=3, experts=6, align=4, seed=12)
    H = 16
    rng = np.random.default_rng(13)
    vals = rng.integers(-50, 50, (rt.max_rows, H))
    eo = torch.tensor(vals, dtype=torch.bfloat16)
    inv = rt.inverse_map.numpy()
    want = np.zeros((rt.tokens, H), np.int64)
    for t in range(rt.tokens):
        for e in range(rt.experts):
            if inv[t, e] >= 0:
                want[t] += vals[inv[t, e]]
    for out_dt, tdt in ((oracle.F32, torch.float32), (oracle.BF16, torch.bfloat16)):
        init = np.zeros((rt.tokens, H), np.float32 if out_dt == oracle.F32 else np.uint16)
        got, err = oracle.unpermute_ordered(bits(eo), oracle.BF16, inv, rt.tokens, init, out_dt)
        assert err == 0
        assert_bits_equal(got, bits(torch.tensor(want, dtype=torch.float64).to(tdt)), "sum")


def test_unpermute_sums_in_increasing_expert_order():
    """Order witness: contributions (1, 2^24, -2^24) from experts 0, 1, 2.
    Ascending order in fp32: (0 + 1) + 2^24 rounds to 2^24 (tie to even),
    then - 2^24 gives 0.  Any order that adds the two large terms first gives 1."""
    eo = torch.tensor([[1.0], [2.0 ** 24], [-(2.0 ** 24)]], dtype=torch.bfloat16)
    inv = np.array([[0, 1, 2], [2, 1, 0]], np.int32)   # token 1: rows in reverse
    got, _ = oracle.unpermute_ordered(bits(eo), oracle.BF16, inv, 2,
                                      np.zeros((2, 1), np.float32), oracle.F32)
    assert got[0, 0] == 0.0
    assert got[1, 0] == 1.0     # (0 + -2^24) + 2^24 + 1


def test_unpermute_untouched_past_valid_tokens_and_bad_entries():
    rt = inputs.routing(tokens=10, top_k=2, experts=4, align=2, seed=14)
    eo = inputs.expert_output_input(rt, 8, seed=15)
    init = np.full((10, 8), 7.0, np.float32)
    got, err = oracle.unpermute_ordered(bits(eo), oracle.BF16, rt.inverse_map.numpy(), 6,
                                        init, oracle.F32)
    assert err == 0 and (got[6:] == 7.0).all() and not np.isnan(got[:6]).any()
    inv = rt.inverse_map.numpy().copy()
    inv[0, np.flatnonzero(inv[0] >= 0)[0]] = rt.max_rows
    _, err = oracle.unpermute_ordered(bits(eo), oracle.BF16, inv, 99, init, oracle.F32)
    assert err == oracle.ERR_COUNT | oracle.ERR_INVERSE


# ------------------------------------------------------ residual add

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_residual_add_bitwise_equals_two_torch_adds(dtype):
    d = inputs.residual_inputs((37, 129), dtype, seed=16)
    want = d["residual"] + (d["expert_output"] + d["shared_expert_output"])
    got = oracle.residual_add(bits(d["expert_output"]), bits(d["shared_expert_output"]),
                              bits(d["residual"]), DT[dtype])
    assert_bits_equal(got, bits(want), "residual add")


def test_residual_add_rounds_expert_sum_first():
    """bf16: e = 1, s = 2^-8 (sum is a tie, rounds to 1), r = 2^-8.
    Two adds: 1 + 2^-8 -> 1 again.  One fused fp32 sum would give 1 + 2^-7."""
    e = torch.tensor([1.0], dtype=torch.bfloat16)
    s = torch.tensor([2.0 ** -8], dtype=torch.bfloat16)
    got = oracle.residual_add(bits(e), bits(s), bits(s), oracle.BF16)
    assert got[0] == bits(torch.tensor([1.0], dtype=torch.bfloat16))[0]
    fused = (e.float() + s.float() + s.float()).to(torch.bfloat16)
    assert float(fused) == 1.0 + 2.0 ** -7


# ------------------------------------------------------ input generators

def test_routing_layout_invariants():
    rt = inputs.routing(tokens=64, top_k=4, experts=8, align=16, seed=17)
    pm = rt.permutation_map.numpy()
    live = pm[pm >= 0]
    assert sorted(live.tolist()) == list(range(64 * 4))
    assert rt.n_used % 16 == 0 and (pm[rt.n_used:] == -1).all()
    inv = rt.inverse_map.numpy()
    assert ((inv >= 0).sum(1) == 4).all()
    for t in range(64):
        for e in np.flatnonzero(inv[t] >= 0):
            assert pm[inv[t, e]] // 4 == t
    # rows grouped by expert, ascending, token order kept inside an expert
    rows = inv[inv >= 0]
    assert np.unique(rows).size == rows.size
    np.testing.assert_allclose(rt.probs.reshape(64, 4).sum(1).numpy(), 1.0, rtol=1e-6)


# ------------------------------------------------------ bounded weighted SwiGLU

@pytest.mark.parametrize("bound_rows,extra", [(37, 0), (20, 5), (0, 0), (50, 0)])
def test_weighted_silu_mul_bounded_vs_torch(bound_rows, extra):
    rows, half_n = 50, 24
    g = torch.Generator().manual_seed(21)
    y = (torch.randn(rows, 2 * half_n, generator=g) * 3).to(torch.bfloat16)
    w = torch.rand(rows, generator=g)
    bound = bound_rows * half_n + extra
    canary = np.full((rows, half_n), 0x1234, np.uint16)
    got, err = oracle.weighted_silu_mul_bounded(bits(y), bits(w), canary, bound)
    assert err == 0
    want = bits((F.silu(y[:, :half_n].float()) * y[:, half_n:].float() * w[:, None])
                .to(torch.bfloat16))
    flat_got, flat_want = got.reshape(-1), want.reshape(-1)
    assert_within_ulp16(flat_got[:bound], flat_want[:bound], 1, what="bounded swiglu")
    assert (flat_got[bound:] == 0x1234).all()


def test_weighted_silu_mul_bounded_clamps_a_bad_bound():
    y = torch.ones(4, 16, dtype=torch.bfloat16)
    out0 = np.zeros((4, 8), np.uint16)
    got, err = oracle.weighted_silu_mul_bounded(bits(y), np.ones(4, np.float32), out0, 10 ** 6)
    assert err == oracle.ERR_COUNT and (got != 0).all()
    _, err = oracle.weighted_silu_mul_bounded(bits(y), np.ones(4, np.float32), out0, -1)
    assert err == oracle.ERR_COUNT


# ------------------------------------------------------ fused epilogue chain

def _chain_inputs(dtype, seed, tokens=30, top_k=3, experts=6, align=4, hidden=40):
    rt = inputs.routing(tokens, top_k, experts, align, seed=seed)
    eo = inputs.expert_output_input(rt, hidden, dtype=dtype, seed=seed + 1)
    pm = rt.permutation_map
    row_probs = torch.where(pm >= 0, rt.probs[pm.clamp(min=0).long()], torch.zeros(()))
    res = inputs.residual_inputs((tokens, hidden), dtype, seed=seed + 2)
    return rt, eo, row_probs.float(), res["shared_expert_output"], res["residual"]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_epilogue_chain_is_the_composition_of_the_three_steps(dtype):
    """Step 1 and 3 by torch (the pages' definitions), step 2 by the pinned
    unpermute oracle: the chain must equal their composition bit for bit."""
    rt, eo, rp, sh, rs = _chain_inputs(dtype, 22)
    dt = DT[dtype]
    kind = "f16" if dtype == torch.float16 else "bf16"
    init = bits(torch.full((rt.tokens, eo.shape[1]), 5.0, dtype=dtype))
    got, err = oracle.epilogue_chain(bits(eo), bits(rp), bits(rt.inverse_map), rt.tokens - 3,
                                     bits(sh), bits(rs), init, dt)
    assert err == 0
    w = (eo.float() * rp[:, None]).to(dtype)             # NaN sentinel rows stay NaN, unread
    routed, _ = oracle.unpermute_ordered(bits(w), dt, bits(rt.inverse_map), rt.tokens - 3,
                                         np.zeros_like(init), dt)
    routed_t = from_bits(routed, dtype)
    want = bits(rs + (routed_t + sh))
    n = rt.tokens - 3
    assert_bits_equal(got[:n], want[:n], "chain", kind=kind)
    assert_bits_equal(got[n:], init[n:], "untouched tokens", kind=kind)


def test_epilogue_chain_exact_integers():
    """Expert rows of small integers with power-of-two probabilities: every
    product and sum is exact, so the chain equals int64 arithmetic."""
    tokens, top_k, experts, hidden = 16, 2, 4, 8
    rt = inputs.routing(tokens, top_k, experts, 2, seed=23)
    rng = np.random.default_rng(24)
    vals = rng.integers(-40, 40, (rt.max_rows, hidden))
    rp = np.where(bits(rt.permutation_map) >= 0, 0.5, 0.0).astype(np.float32)
    sh = rng.integers(-10, 10, (tokens, hidden))
    rs = rng.integers(-10, 10, (tokens, hidden))
    f = lambda a: bits(torch.tensor(a, dtype=torch.float32))      # noqa: E731
    got, _ = oracle.epilogue_chain(f(vals), rp, bits(rt.inverse_map), tokens, f(sh), f(rs),
                                   np.zeros((tokens, hidden), np.float32), oracle.F32)
    inv = bits(rt.inverse_map)
    want = rs + sh + np.array([[sum(vals[inv[t, e], h] for e in range(experts) if inv[t, e] >= 0)
                                for h in range(hidden)] for t in range(tokens)]) * 0.5
    np.testing.assert_array_equal(got, want.astype(np.float32))


# ------------------------------------------------ SwiGLU in fp16 and fp32

def _swiglu_f64_parts(x64, p64, limit):
    inter = x64.shape[1] // 2
    g, u = x64[:, :inter], x64[:, inter:]
    gc = torch.clamp(g, max=limit)
    uc = torch.clamp(u, -limit, limit)
    sg = torch.sigmoid(gc)
    return g, u, gc, uc, sg


@pytest.mark.parametrize("limit", [7.0, float("inf")])
def test_swiglu_fp16_vs_float64_autograd(limit):
    """fp16 storage: forward and grad_x within one fp16 ulp of the float64
    library chain rounded once to fp16; grad_probs within the sum tolerance."""
    d = inputs.swiglu_inputs(40, 72, sigma=3.0, limit=7.0, plant_ties=True, seed=25)
    x16 = d["x"].to(torch.float16)
    gy16 = d["grad_y"].to(torch.float16)
    p = bits(d["probs"])
    y = oracle.swiglu_clamped_fwd(bits(x16), p, limit, oracle.F16)
    assert_within_ulp16(y, bits(_swiglu_ref64_any(x16, p, limit, torch.float16)), 1, kind="f16",
                        what="fp16 fwd")
    gx, gp, gabs = oracle.swiglu_clamped_bwd(bits(x16), p, bits(gy16), limit, oracle.F16)
    xg = x16.double().requires_grad_(True)
    pg = torch.from_numpy(p).double().reshape(-1, 1).requires_grad_(True)
    g_, u_, gc, uc, _ = _swiglu_f64_parts(xg, pg, limit)
    (F.silu(gc) * uc * pg).backward(gy16.double())
    assert_within_ulp16(gx, bits(xg.grad.to(torch.float16)), 1, kind="f16", what="fp16 grad_x")
    assert_sum_close(gp, pg.grad.reshape(-1).numpy(), gabs, 1e-6, "fp16 grad_probs")


def _swiglu_ref64_any(x, p, limit, dtype):
    x64 = x.double()
    inter = x64.shape[1] // 2
    y = F.silu(torch.clamp(x64[:, :inter], max=limit)) * torch.clamp(x64[:, inter:], -limit, limit)
    return (y * torch.from_numpy(np.asarray(p)).double().reshape(-1, 1)).to(dtype)


def test_swiglu_fp32_vs_float64_autograd():
    """fp32 storage: every output within 2^-20 of the float64 value relative to
    the magnitude of its terms (for d_gate: |dy p uc| sigma (1 + |gc| (1 - sigma)),
    which bounds the cancellation in silu')."""
    limit = 7.0
    g = torch.Generator().manual_seed(26)
    x = torch.randn(30, 2 * 50, generator=g) * 4
    x[0, 0], x[1, 50] = limit, -limit                                  # ties stay inclusive
    dy = torch.randn(30, 50, generator=g)
    p = torch.rand(30, generator=g)
    y = oracle.swiglu_clamped_fwd(x.numpy(), p.numpy(), limit, oracle.F32)
    ref = _swiglu_ref64_any(x, p.numpy(), limit, torch.float64).numpy()
    assert (np.abs(y - ref) <= 2 ** -20 * np.abs(ref) + 1e-30).all()
    gx, gp, gabs = oracle.swiglu_clamped_bwd(x.numpy(), p.numpy(), dy.numpy(), limit, oracle.F32)
    xg = x.double().requires_grad_(True)
    pg = p.double().reshape(-1, 1).requires_grad_(True)
    _, _, gc, uc, sg = _swiglu_f64_parts(xg, pg, limit)
    (F.silu(gc) * uc * pg).backward(dy.double())
    with torch.no_grad():
        a = (dy.double() * pg).abs()
        scale_g = a * uc.abs() * sg * (1 + gc.abs() * (1 - sg))
        scale_u = a * (gc * sg).abs()
    err = np.abs(gx - xg.grad.numpy())
    scale = np.concatenate([scale_g.numpy(), scale_u.numpy()], 1)
    assert (err <= 2 ** -20 * scale + 1e-30).all()
    assert gx[0, 0] != 0 and gx[1, 50] != 0
    assert_sum_close(gp, pg.grad.reshape(-1).numpy(), gabs, 1e-6, "fp32 grad_probs")


@pytest.mark.parametrize("p_dtype", [torch.bfloat16, torch.float16])
def test_router_weight_low_precision_probs_vs_torch(p_dtype):
    """bf16 / fp16 routing probabilities: the forward widens them exactly
    (probs.float()) -- bitwise equal to torch; the backward's grad_x likewise
    and grad_probs is torch autograd's fp32 sum (cast to the probs dtype by
    the caller of the oracle)."""
    d = inputs.router_weight_inputs(24, 200, seed=27)
    probs = d["probs"].to(p_dtype)
    x = d["x"].clone().requires_grad_(True)
    p = probs.clone().requires_grad_(True)
    out = (x.float() * p.float()).to(torch.bfloat16)
    got = oracle.router_weight_fwd(bits(d["x"]), oracle.BF16, bits(probs), oracle.BF16,
                                   DT[p_dtype])
    assert_bits_equal(got, bits(out), "fwd with low-precision probs")
    out.backward(d["grad_out"])
    gx, gp, gabs = oracle.router_weight_bwd(bits(d["grad_out"]), oracle.BF16, bits(d["x"]),
                                            oracle.BF16, bits(probs), DT[p_dtype])
    assert_bits_equal(gx, bits(x.grad), "grad_x")
    # torch rounds its fp32 sum to the probs dtype: within one ulp of that dtype
    want = p.grad.reshape(-1).double().numpy()
    rel = 2.0 ** -7 if p_dtype == torch.bfloat16 else 2.0 ** -10
    assert (np.abs(gp - want) <= rel * np.abs(want) + 1e-5 * gabs).all()


# ------------------------------------------------- rank-order reduce-scatter

def _rs(inputs_list, in_dt, rank, offsets, ep_tokens, local, hidden, out_dt, init=0):
    out0 = np.full((local, hidden), init, oracle._storage_np(out_dt))
    return oracle.ordered_reduce_scatter_v(inputs_list, in_dt, rank, offsets, ep_tokens, out0,
                                           out_dt)


def test_reduce_scatter_exact_integers_pick_the_rank_rows():
    """fp32 buffers x_q[g, h] = (q + 1) * (g * hidden + h + 1): every partial
    sum is an integer below 2^24, so the exact sum is (1 + ... + W) * (g*H + h
    + 1) for whichever rows g were read.  A wrong offset, a dropped or repeated
    rank, or a transposed index changes it."""
    world, hidden, counts = 4, 6, [3, 0, 5, 2]
    offsets = np.concatenate([[0], np.cumsum(counts)[:-1]]).astype(np.int32)
    total = int(sum(counts))
    cap = total + 3
    g = np.arange(cap, dtype=np.float64)[:, None] * hidden + np.arange(hidden) + 1
    bufs = [((q + 1) * g).astype(np.float32) for q in range(world)]
    for rank in range(world):
        out, err = _rs(bufs, oracle.F32, rank, offsets, total, counts[rank], hidden, oracle.F32)
        assert err == 0
        rows = offsets[rank] + np.arange(counts[rank])
        want = world * (world + 1) // 2 * g[rows]
        assert np.array_equal(out.astype(np.float64), want), rank


def test_reduce_scatter_adds_in_rank_order():
    """fp32 witness of the order: 2^24 + 1 rounds back to 2^24 (ties to even),
    so ((2^24 + 1) + 1) = 2^24 while ((1 + 1) + 2^24) = 2^24 + 2."""
    big, one = np.float32(2.0 ** 24), np.float32(1.0)
    cols = [np.array([[big, one]], np.float32), np.array([[one, one]], np.float32),
            np.array([[one, big]], np.float32)]
    out, err = _rs(cols, oracle.F32, 0, [0, 0, 0], 1, 1, 2, oracle.F32)
    assert err == 0
    assert out[0, 0] == 2.0 ** 24 and out[0, 1] == 2.0 ** 24 + 2


def test_reduce_scatter_rounds_once_at_the_end():
    """bf16 witness: 1 + 2^-8 + 2^-8 = 1 + 2^-7 is a bf16 value (0x3F81), but
    rounding after each add (1 + 2^-8 is a tie -> 1) would give 1.0 (0x3F80)."""
    vals = [1.0, 2.0 ** -8, 2.0 ** -8]
    bufs = [oracle.bf16_from_f32(np.array([v], np.float32)).reshape(1, 1) for v in vals]
    out, _ = _rs(bufs, oracle.BF16, 0, [0, 0, 0], 1, 1, 1, oracle.BF16)
    assert int(out[0, 0]) == 0x3F81


@pytest.mark.parametrize("in_dtype,out_dtype", [(torch.bfloat16, torch.bfloat16),
                                                (torch.float16, torch.float32),
                                                (torch.float32, torch.bfloat16)])
def test_reduce_scatter_two_ranks_vs_torch(in_dtype, out_dtype):
    """W = 2: one fp32 add and one rounding, which torch computes as
    (a.float() + b.float()).to(out); W = 1: a plain dtype conversion."""
    odt = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}
    gen = torch.Generator().manual_seed(11)
    a = (torch.randn(40, 24, generator=gen) * 3).to(in_dtype)
    b = (torch.randn(40, 24, generator=gen) * 3).to(in_dtype)
    out, err = _rs([bits(a), bits(b)], odt[in_dtype], 1, [0, 17], 40, 20, 24, odt[out_dtype])
    assert err == 0
    assert_bits_equal(out, bits((a.float() + b.float()).to(out_dtype)[17:37]), "W=2")
    one, _ = _rs([bits(a)], odt[in_dtype], 0, [5], 40, 30, 24, odt[out_dtype])
    assert_bits_equal(one, bits(a.to(out_dtype)[5:35]), "W=1")


def test_reduce_scatter_within_the_fp32_error_bound():
    """Random bf16 partials, W = 8: the result is within the textbook bound of a
    recursive fp32 sum, (W - 1) u32 sum|x| (u32 = 2^-24), of the exact float64
    sum -- before the final rounding, here to fp32 so none is added."""
    world, cap, hidden = 8, 64, 33
    gen = torch.Generator().manual_seed(12)
    ts = [(torch.randn(cap, hidden, generator=gen) * 10.0 ** (q % 3)).to(torch.bfloat16)
          for q in range(world)]
    out, err = _rs([bits(t) for t in ts], oracle.BF16, 3, [0, 8, 16, 24, 32, 40, 48, 56], 64, 8,
                   hidden, oracle.F32)
    assert err == 0
    x = np.stack([t.double().numpy()[24:32] for t in ts])
    exact, mag = x.sum(0), np.abs(x).sum(0)
    assert (np.abs(out - exact) <= (world - 1) * 2.0 ** -24 * mag + 1e-300).all()


def test_reduce_scatter_bounds():
    """Rows past ep_tokens are neither read nor written; an ep_tokens beyond
    the buffers is clamped to them; both set the count error."""
    cap, hidden = 10, 4
    bufs = [np.full((cap, hidden), q + 1.0, np.float32) for q in range(2)]
    out, err = _rs(bufs, oracle.F32, 1, [0, 6], 8, 4, hidden, oracle.F32, init=-7.0)
    assert err == oracle.ERR_COUNT
    assert (out[:2] == 3.0).all() and (out[2:] == -7.0).all()
    out, err = _rs(bufs, oracle.F32, 1, [0, 6], 12, 4, hidden, oracle.F32, init=-7.0)
    assert err == oracle.ERR_COUNT and (out == 3.0).all()
    out, err = _rs(bufs, oracle.F32, 0, [-1, 6], 10, 2, hidden, oracle.F32, init=-7.0)
    assert err == oracle.ERR_COUNT and (out[0] == -7.0).all() and (out[1] == 3.0).all()


# ------------------------------------------------ EP combine (unpermute + RS)

@pytest.mark.parametrize("partial_dtype,out_dtype", [(torch.bfloat16, torch.bfloat16),
                                                     (torch.float32, torch.bfloat16),
                                                     (torch.float32, torch.float32)])
def test_ep_combine_is_the_composition_of_the_two_steps(partial_dtype, out_dtype):
    """Per rank, the oracle's unpermute into a partial block, then its
    rank-order reduce-scatter (both pinned above) -- called one after another
    here -- give the combined function's bits."""
    odt = {torch.bfloat16: oracle.BF16, torch.float32: oracle.F32}
    case = inputs.ep_combine_inputs(3, 40, 3, 4, 4, 24, seed=21)
    eos = [bits(e) for e in case.expert_outputs]
    invs = [bits(i) for i in case.inverse_maps]
    blocks = []
    for q in range(3):
        blk, err = oracle.unpermute_ordered(eos[q], oracle.BF16, invs[q], case.tokens,
                                            np.zeros((case.tokens, 24),
                                                     oracle._storage_np(odt[partial_dtype])),
                                            odt[partial_dtype])
        assert err == 0
        blocks.append(blk)
    offs = case.rank_token_offset.numpy()
    for rank in range(3):
        init = np.zeros((case.counts[rank], 24), oracle._storage_np(odt[out_dtype]))
        want, err = oracle.ordered_reduce_scatter_v(blocks, odt[partial_dtype], rank, offs,
                                                    case.tokens, init, odt[out_dtype])
        got, err2 = oracle.unpermute_reduce_scatter(eos, oracle.BF16, invs, case.tokens, rank,
                                                    offs, odt[partial_dtype], init, odt[out_dtype])
        assert err == err2 == 0
        assert_bits_equal(got, want, f"rank {rank}")


def test_ep_combine_exact_integers():
    """fp32 expert rows holding small integers: every sum is exact, so the
    result is the integer sum over all ranks' experts of the token's rows,
    computed here by brute force in int64 from the routing."""
    world, tokens, top_k, epr, H = 4, 30, 3, 2, 5
    case = inputs.ep_combine_inputs(world, tokens, top_k, epr, 2, H, dtype=torch.float32,
                                    seed=22)
    rng = np.random.default_rng(0)
    eos = [rng.integers(-50, 50, (case.max_rows, H)).astype(np.float32) for _ in range(world)]
    invs = [bits(i) for i in case.inverse_maps]
    offs = case.rank_token_offset.numpy()
    for rank in range(world):
        got, err = oracle.unpermute_reduce_scatter(
            eos, oracle.F32, invs, tokens, rank, offs, oracle.F32,
            np.zeros((case.counts[rank], H), np.float32), oracle.F32)
        assert err == 0
        for t in range(case.counts[rank]):
            g = offs[rank] + t
            want = np.zeros(H, np.int64)
            for q in range(world):
                for e in range(epr):
                    r = invs[q][g, e]
                    if r >= 0:
                        want += eos[q][r].astype(np.int64)
            assert np.array_equal(got[t].astype(np.int64), want), (rank, t)


def test_ep_combine_rounds_each_rank_partial():
    """bf16 partials: rank 0's experts give 1 + 2^-8 (a tie: rounds to 1), rank 1
    gives 2^-8, so the combined fp32 result is 1 + 2^-8; with fp32 partials it
    is 1 + 2^-7.  One token, one column."""
    vals = [[1.0, 2.0 ** -8], [2.0 ** -8, 0.0]]
    eos = [np.array([[v] for v in vals[q]], np.float32) for q in range(2)]
    invs = [np.array([[0, 1]], np.int32), np.array([[0, -1]], np.int32)]
    out_b, _ = oracle.unpermute_reduce_scatter(eos, oracle.F32, invs, 1, 0, [0, 1], oracle.BF16,
                                               np.zeros((1, 1), np.float32), oracle.F32)
    out_f, _ = oracle.unpermute_reduce_scatter(eos, oracle.F32, invs, 1, 0, [0, 1], oracle.F32,
                                               np.zeros((1, 1), np.float32), oracle.F32)
    assert out_b[0, 0] == 1.0 + 2.0 ** -8 and out_f[0, 0] == 1.0 + 2.0 ** -7


# ------------------------------------------------------------ identities

@pytest.mark.parametrize("x_dtype,out_dtype", [(torch.bfloat16, torch.bfloat16),
                                               (torch.float32, torch.bfloat16),
                                               (torch.bfloat16, torch.float16)])
def test_router_weight_unit_probs_is_a_cast(x_dtype, out_dtype):
    """probs = 1 is the identity weighting: x * 1 is exact, so the forward is a
    plain dtype conversion of x (torch's), and grad_x one of grad_out."""
    odt = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}
    g = torch.Generator().manual_seed(31)
    x = (torch.randn(33, 70, generator=g) * 5).to(x_dtype)
    ones = np.ones(33, np.float32)
    out = oracle.router_weight_fwd(bits(x), odt[x_dtype], ones, odt[out_dtype])
    assert_bits_equal(out, bits(x.to(out_dtype)), "fwd with unit probs",
                      kind="f16" if out_dtype == torch.float16 else "bf16")
    gx, _, _ = oracle.router_weight_bwd(bits(x), odt[x_dtype], None, odt[out_dtype], ones)
    assert_bits_equal(gx, bits(x.to(out_dtype)), "grad_x with unit probs",
                      kind="f16" if out_dtype == torch.float16 else "bf16")


def test_unpermute_single_expert_is_a_copy():
    """A token routed to one local expert gets that expert row exactly (+0 + x
    is x for every x but -0), converted by torch to the output dtype."""
    g = torch.Generator().manual_seed(32)
    eo = (torch.randn(10, 24, generator=g) * 3).to(torch.bfloat16)
    inv = np.full((6, 4), -1, np.int32)
    rows = [7, 2, 9, 0, 5, 3]
    for t, r in enumerate(rows):
        inv[t, t % 4] = r
    for odt, tdt in ((oracle.BF16, torch.bfloat16), (oracle.F32, torch.float32)):
        out, err = oracle.unpermute_ordered(bits(eo), oracle.BF16, inv, 6,
                                            np.zeros((6, 24), oracle._storage_np(odt)), odt)
        assert err == 0
        want = eo[torch.tensor(rows)].to(tdt)
        want = torch.where(want == 0, torch.zeros((), dtype=tdt), want)   # -0 becomes +0
        assert_bits_equal(out, bits(want), f"copy to {tdt}")


# --------------------------------------------------- seeded random sweeps

@pytest.mark.parametrize("case", range(8))
def test_random_shapes_residual_and_router_weight_vs_torch(case):
    """Random shapes and dtypes: the residual add equals torch's two adds and
    the router-weight forward torch's fp32 multiply and cast, bit for bit."""
    rng = np.random.default_rng(100 + case)
    dts = [torch.bfloat16, torch.float16, torch.float32]
    odt = {torch.bfloat16: oracle.BF16, torch.float16: oracle.F16, torch.float32: oracle.F32}
    g = torch.Generator().manual_seed(case)
    dt = dts[case % 3]
    shape = (int(rng.integers(1, 50)), int(rng.integers(1, 90)))
    e, s_, r = ((torch.randn(*shape, generator=g) * 4).to(dt) for _ in range(3))
    assert_bits_equal(oracle.residual_add(bits(e), bits(s_), bits(r), odt[dt]),
                      bits(r + (e + s_)) if dt == torch.float32 else
                      bits((r.float() + (e.float() + s_.float()).to(dt).float()).to(dt)),
                      "residual", kind="f16" if dt == torch.float16 else "bf16")
    x_dt, o_dt = dts[int(rng.integers(0, 3))], dts[int(rng.integers(0, 3))]
    x = (torch.randn(*shape, generator=g) * 3).to(x_dt)
    p = torch.rand(shape[0], 1, generator=g) + 0.01
    assert_bits_equal(oracle.router_weight_fwd(bits(x), odt[x_dt], bits(p), odt[o_dt]),
                      bits((x.float() * p).to(o_dt)), "router weight",
                      kind="f16" if o_dt == torch.float16 else "bf16")
