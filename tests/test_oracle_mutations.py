"""The oracle's pins catch plausible mistakes (not gpu).

Each case plants one mistake in a copy of oracle/moe_oracle.c (a dropped
term, a wrong sign or index, a swapped operand, a wrong mask boundary, a lost
rounding step), builds it with gcc into a temporary library, swaps it in for
the oracle and runs the pins that should notice: at least one must fail.
The real oracle is restored afterwards and is never modified."""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

# (id, text in the source, replacement, pins expected to fail)
MUTATIONS = [
    ("swap_gate_up", "float g = load_as_f32(x, dt, r * ld_x + j);\n            float u = "
     "load_as_f32(x, dt, r * ld_x + inter + j);\n            float gc = clamp_max_f32(g, limit);"
     "\n            float uc = clamp_f32(u, -limit, limit);\n            float s = gc * sigmoid_f32(gc);"
     "\n            float v = s * uc;",
     "float u = load_as_f32(x, dt, r * ld_x + j);\n            float g = "
     "load_as_f32(x, dt, r * ld_x + inter + j);\n            float gc = clamp_max_f32(g, limit);"
     "\n            float uc = clamp_f32(u, -limit, limit);\n            float s = gc * sigmoid_f32(gc);"
     "\n            float v = s * uc;",
     ["test_swiglu_fwd_vs_float64_library_chain"]),
    ("sigmoid_sign", "return 1.0f / (1.0f + expf(-z));", "return 1.0f / (1.0f + expf(z));",
     ["test_swiglu_fwd_closed_forms"]),
    ("drop_dsilu_term", "float dsilu = sg * (1.0f + gc * (1.0f - sg));", "float dsilu = sg;",
     ["test_swiglu_bwd_vs_float64_autograd", "test_swiglu_bwd_vs_float64_finite_differences"]),
    ("exclusive_gate_mask", "int gate_in = (g <= limit);", "int gate_in = (g < limit);",
     ["test_swiglu_bwd_inclusive_masks_at_planted_ties"]),
    ("exclusive_up_mask", "int up_in = (u >= -limit) && (u <= limit);",
     "int up_in = (u > -limit) && (u < limit);",
     ["test_swiglu_bwd_inclusive_masks_at_planted_ties"]),
    ("probs_grad_wrong_operand", "float t = dy * (s * uc);", "float t = dy * (s * p);",
     ["test_swiglu_bwd_vs_float64_autograd"]),
    ("bf16_truncates", "u += 0x7fffu + ((u >> 16) & 1u);", "u += 0u;",
     ["test_bf16_rounding_matches_torch"]),
    ("f16_ties_away", "if (rem > 0x1000u || (rem == 0x1000u && (q & 1u))) q++;",
     "if (rem >= 0x1000u) q++;", ["test_f16_rounding_matches_numpy"]),
    ("rw_grad_probs_uses_p", "float t = g * load_as_f32(x, x_dt, r * hidden + h);",
     "float t = g * p;", ["test_router_weight_bwd_vs_torch_autograd"]),
    ("sqrelu_single_rounding", "float sq = round_to_dtype(rl * rl, ORC_BF16);",
     "float sq = rl * rl;", ["test_sqrelu_rounding_witness"]),
    ("clamp_scale_dropped", "float z = clamp_scale * tanhf(xv / clamp_scale);",
     "float z = tanhf(xv / clamp_scale);", ["test_act_permuted_brute_force"]),
    ("unpermute_descending", "for (int32_t e = 0; e < num_local_experts; ++e) {",
     "for (int32_t e = num_local_experts - 1; e >= 0; --e) {",
     ["test_unpermute_sums_in_increasing_expert_order"]),
    ("bounded_drops_weight", "float v = (s * u) * weights[r];", "float v = s * u;",
     ["test_weighted_silu_mul_bounded_vs_torch"]),
    ("bounded_off_by_one", "for (int64_t e = 0; e < n; ++e) {\n        int64_t r = e / half_n",
     "for (int64_t e = 0; e <= n && e < rows * half_n; ++e) {\n        int64_t r = e / half_n",
     ["test_weighted_silu_mul_bounded_vs_torch"]),
    ("rs_reverse_rank_order",
     "float acc = load_as_f32(inputs[0], in_dt, g * hidden + h);\n"
     "            for (int32_t q = 1; q < world; ++q)\n"
     "                acc = acc + load_as_f32(inputs[q], in_dt, g * hidden + h);",
     "float acc = load_as_f32(inputs[world - 1], in_dt, g * hidden + h);\n"
     "            for (int32_t q = world - 2; q >= 0; --q)\n"
     "                acc = acc + load_as_f32(inputs[q], in_dt, g * hidden + h);",
     ["test_reduce_scatter_adds_in_rank_order"]),
    ("rs_first_rank_offset", "const int64_t first = rank_token_offset[rank];",
     "const int64_t first = rank_token_offset[0];",
     ["test_reduce_scatter_exact_integers_pick_the_rank_rows"]),
    ("rs_drops_last_rank", "for (int32_t q = 1; q < world; ++q)",
     "for (int32_t q = 1; q < world - 1; ++q)",
     ["test_reduce_scatter_exact_integers_pick_the_rank_rows"]),
    ("rs_rounds_each_add",
     "acc = acc + load_as_f32(inputs[q], in_dt, g * hidden + h);",
     "acc = round_to_dtype(acc + load_as_f32(inputs[q], in_dt, g * hidden + h), out_dt);",
     ["test_reduce_scatter_rounds_once_at_the_end"]),
    ("combine_first_rank_map_for_all",
     "err |= orc_unpermute_ordered(expert_outputs[q], eo_dt, max_rows, inverse_maps[q],",
     "err |= orc_unpermute_ordered(expert_outputs[q], eo_dt, max_rows, inverse_maps[0],",
     ["test_ep_combine_exact_integers"]),
    ("chain_swaps_shared_and_residual",
     "orc_residual_add(routed, shared_expert_output, residual, out, n * hidden, dt);",
     "orc_residual_add(routed, residual, shared_expert_output, out, n * hidden, dt);",
     ["test_epilogue_chain_is_the_composition_of_the_three_steps"]),
    ("residual_single_rounding", "float t = round_to_dtype(e + s, dt);", "float t = e + s;",
     ["test_residual_add_rounds_expert_sum_first",
      "test_residual_add_bitwise_equals_two_torch_adds"]),
]


def _call_pin(name):
    fn = getattr(pins, name)
    import inspect
    params = inspect.signature(fn).parameters
    mark_args = {}
    for m in getattr(fn, "pytestmark", []):
        if m.name == "parametrize":
            argnames, values = m.args
            names = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) \
                else list(argnames)
            mark_args[tuple(names)] = values
    # run every parametrization; report True if any fails
    combos = [{}]
    for names, values in mark_args.items():
        combos = [dict(c, **dict(zip(names, v if len(names) > 1 else (v,))))
                  for c in combos for v in values]
    for c in combos:
        try:
            fn(**{k: v for k, v in c.items() if k in params})
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("mid,old,new,expect", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, mid, old, new, expect):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {mid} not found exactly once"
    mutated = tmp_path / "moe_oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", *oracle._CFLAGS, "-o", str(so), str(mutated), "-lm"], check=True)
    real = oracle._lib()
    try:
        oracle._LIB = oracle.load(str(so))
        caught = [name for name in expect if _call_pin(name)]
    finally:
        oracle._LIB = real
    assert caught, f"planted mistake {mid} passed every pin in {expect}"
