#!/usr/bin/env python
"""Clamped-SwiGLU fwd+bwd throughput on B200 inside the MoE expert-epilogue pass.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole epilogue over one batch of seeded synthetic
inputs that are resident in HBM before timing starts:

    clamped SwiGLU fwd and bwd      rows 65536 (8192 tokens x top-8), inter 2048, L 10
    router-weight multiply fwd/bwd  [16384, 7168] bf16, fp32 probs, save_x on
    permuted activation x3          8192 tokens, top-8 of 64 experts, 128-row alignment,
                                    width 1536: SQRELU, SQRELU_CLAMP (scale 7), SWIGLU,
                                    zero padding on
    fixed-order unpermute           -> [8192, 4096] bf16
    residual add                    [32768, 7168] bf16; its expert_output's first
                                    16384 rows are the router-weight forward's output

The headline (`value`, `ms_per_step`) is the metric the line names: the
clamped-SwiGLU forward + backward (the two launches run back to back at the
start of every step) in achieved HBM GB/s = their algorithmic bytes over the
time between a CUDA event recorded before the forward and one recorded after
the backward, summed over all K timed steps (one more event between the two
launches splits the time per kernel); max over ranks.  The whole step is
reported under `step` (its bytes over the time of the K steps).  The other
kernels get CUDA events around each launch on every 10th timed step (event
records between kernels stop programmatic launch overlap).  Every kernel's
working set exceeds the 126 MB L2, so no flush is needed between steps.
Multi-GPU runs (torchrun) are weak scaling: each rank runs the full step on its
own inputs; the data path has no collective, the barrier and the max of the
timings are the only ones.  With N > 1 the line also carries `collectives`:
the rank-order reduce-scatter and the EP combine across the N ranks over
their peer-mapped buffers, timed after the step.

The line also carries `e2e` (the same step through the public API with every
input copied from pinned host memory and every output copied back inside the
timed region, pipelined), `configs` (the workload's other configurations:
the small SwiGLU, the router-weight output-dtype / save_x variants, the
residual add in three dtypes alone and chained after the router-weight
forward, the fp32-output unpermute), `next_rows` (the bounded SwiGLU, the
fused chain, the reduce-scatter, the EP combine, and the other storage dtypes:
the SwiGLU in fp16 and fp32, the router weight with bf16 and fp16
probabilities; timed after the step),
`clocks`, `roofline` and `cpu_baseline` (the CPU oracle, one core and all
cores).  `--impl reference` times the CPU oracle alone on every host core.
"""
from __future__ import annotations

import argparse
import contextlib
import datetime
import hashlib
import json
import os
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "clamped-SwiGLU fwd+bwd achieved HBM GB/s and % of B200 peak; rows/s"
FALLBACK_HBM_GBS = 6650.0

# ---------------------------------------------------------------- workload

SWIGLU = dict(rows=65536, inter=2048, limit=10.0, sigma=3.0)
ROUTER = dict(rows=16384, hidden=7168)
PERMUTED = dict(tokens=8192, top_k=8, experts=64, align=128, width=1536, hidden=4096, scale=7.0)
RESIDUAL = dict(rows=32768, hidden=7168)


def scaled(scale: float) -> dict:
    """The workload with every op's row (token) count multiplied by `scale`
    (1.0 = the benchmark; smaller scales serve short profiler captures)."""
    f = lambda n, m=8: max(m, int(n * scale) // m * m)  # noqa: E731
    return {"swiglu": dict(SWIGLU, rows=f(SWIGLU["rows"])),
            "router": dict(ROUTER, rows=f(ROUTER["rows"])),
            "permuted": dict(PERMUTED, tokens=f(PERMUTED["tokens"])),
            "residual": dict(RESIDUAL, rows=f(RESIDUAL["rows"]))}


WORKLOAD_NAME = ("moe_expert_epilogue_pass: clamped SwiGLU fwd+bwd rows=65536 inter=2048 L=10; "
                 "router-weight fwd+bwd [16384,7168]; permuted SQRELU/SQRELU_CLAMP/SWIGLU + "
                 "ordered unpermute (8192 tok, top-8 of 64, align 128, width 1536, hidden 4096); "
                 "residual add [32768,7168]; all bf16 with fp32 probs")
HEADLINE_NAME = ("clamped SwiGLU fwd+bwd: rows=65536 (8192 tokens x top-8), inter=2048, L=10, "
                 "x bf16 [65536, 4096] ~N(0, 3^2), fp32 top-8 softmax probs, grad_y bf16 ~N(0,1)")


def algorithmic_bytes(n_used: int, scale: float = 1.0) -> dict:
    """Minimal bytes per launch: each input byte read once, each output byte
    written once; padding rows count as written (zero padding), never as read."""
    w = scaled(scale)
    R, I = w["swiglu"]["rows"], SWIGLU["inter"]
    Rr, H = w["router"]["rows"], ROUTER["hidden"]
    live = w["permuted"]["tokens"] * PERMUTED["top_k"]
    W = PERMUTED["width"]
    T, E, Hu = w["permuted"]["tokens"], PERMUTED["experts"], PERMUTED["hidden"]
    meta = 4 * n_used + 4 * live          # permutation map rows + gathered probs
    return {
        "swiglu_fwd": R * (2 * I * 2 + 4 + I * 2),
        "swiglu_bwd": R * (2 * I * 2 + I * 2 + 4 + 2 * I * 2 + 4),
        "router_weight_fwd": Rr * H * 2 * 2 + Rr * 4,
        "router_weight_bwd": Rr * H * 2 * 3 + Rr * 8,
        "act_sqrelu": live * W * 2 + n_used * W * 2 + meta,
        "act_sqrelu_clamp": live * W * 2 + n_used * W * 2 + meta,
        "act_swiglu": live * 2 * W * 2 + n_used * W * 2 + meta,
        "unpermute": live * Hu * 2 + T * E * 4 + T * Hu * 2,
        "residual_add": 4 * w["residual"]["rows"] * RESIDUAL["hidden"] * 2,
    }


def rows_per_launch(scale: float = 1.0) -> dict:
    """Rows (tokens) one launch processes, for rows/s."""
    w = scaled(scale)
    return {"swiglu_fwd": w["swiglu"]["rows"], "swiglu_bwd": w["swiglu"]["rows"],
            "router_weight_fwd": w["router"]["rows"], "router_weight_bwd": w["router"]["rows"],
            "act_sqrelu": None, "act_sqrelu_clamp": None, "act_swiglu": None,
            "unpermute": w["permuted"]["tokens"], "residual_add": w["residual"]["rows"]}

KERNEL_SOURCES = {
    "swiglu_fwd": "swiglu_clamped.cu", "swiglu_bwd": "swiglu_clamped.cu",
    "router_weight_fwd": "router_weight.cu", "router_weight_bwd": "router_weight.cu",
    "act_sqrelu": "act_permuted.cu", "act_sqrelu_clamp": "act_permuted.cu",
    "act_swiglu": "act_permuted.cu", "unpermute": "unpermute_ordered.cu",
    "residual_add": "residual_add.cu",
}


GROUPS = {  # kernel -> the input group it needs
    "swiglu_fwd": "swiglu", "swiglu_bwd": "swiglu",
    "router_weight_fwd": "router", "router_weight_bwd": "router",
    "act_sqrelu": "act", "act_sqrelu_clamp": "act", "act_swiglu": "act",
    "unpermute": "unpermute", "residual_add": "residual",
}
# The clamped SwiGLU's forward and backward open every step back to back: the
# headline brackets the two with one event pair.
ORDER = ["swiglu_fwd", "swiglu_bwd", "router_weight_fwd", "act_sqrelu", "act_sqrelu_clamp",
         "act_swiglu", "unpermute", "residual_add", "router_weight_bwd"]
HEAD = ("swiglu_fwd", "swiglu_bwd")


class Batch:
    """All inputs and outputs of one step (or of the selected kernels), on one device."""

    def __init__(self, device, seed, scale=1.0, kernels=None):
        from moe_expert_epilogue_b200 import inputs
        self.scale = scale
        self.names = [k for k in ORDER if kernels is None or k in kernels]
        groups = {GROUPS[k] for k in self.names}
        w = scaled(scale)
        gen_dev = device if device.type == "cuda" else "cpu"
        z = lambda *s, dt=torch.bfloat16: torch.empty(*s, dtype=dt, device=device)  # noqa: E731
        self.inputs, self.outputs = [], []
        W = PERMUTED["width"]
        # routing metadata is always drawn: its n_used enters the byte count
        rt = inputs.routing(w["permuted"]["tokens"], PERMUTED["top_k"], PERMUTED["experts"],
                            PERMUTED["align"], seed=seed + 2, device=gen_dev)
        self.rt = rt
        if "swiglu" in groups:
            sw = inputs.swiglu_inputs(w["swiglu"]["rows"], SWIGLU["inter"], sigma=SWIGLU["sigma"],
                                      probs="topk_softmax", seed=seed, device=gen_dev)
            self.sw_x, self.sw_p, self.sw_gy = sw["x"], sw["probs"], sw["grad_y"]
            R, I = w["swiglu"]["rows"], SWIGLU["inter"]
            self.sw_y, self.sw_gx, self.sw_gp = z(R, I), z(R, 2 * I), z(R, 1, dt=torch.float32)
            self.inputs += ["sw_x", "sw_p", "sw_gy"]
            self.outputs += ["sw_y", "sw_gx", "sw_gp"]
        if "router" in groups:
            rw = inputs.router_weight_inputs(w["router"]["rows"], ROUTER["hidden"], seed=seed + 1,
                                             device=gen_dev)
            self.rw_x, self.rw_p, self.rw_g = rw["x"], rw["probs"], rw["grad_out"]
            Rr = w["router"]["rows"]
            self.rw_gx, self.rw_gp = z(Rr, ROUTER["hidden"]), z(Rr, 1, dt=torch.float32)
            self.inputs += ["rw_x", "rw_p", "rw_g"]
            self.outputs += ["rw_gx", "rw_gp"]
        if "act" in groups:
            self.act_x = inputs.permuted_activation_input(rt, W, swiglu=False, seed=seed + 3,
                                                          device=gen_dev)
            self.act_x2 = inputs.permuted_activation_input(rt, W, swiglu=True, seed=seed + 4,
                                                           device=gen_dev)
            self.act_o1, self.act_o2, self.act_o3 = (z(rt.max_rows, W) for _ in range(3))
            self.inputs += ["act_x", "act_x2"]
            self.outputs += ["act_o1", "act_o2", "act_o3"]
        if "act" in groups or "unpermute" in groups:
            self.pmap, self.probs = rt.permutation_map, rt.probs
            self.n_used = torch.tensor([rt.n_used], dtype=torch.int32, device=gen_dev)
            self.inv = rt.inverse_map
            self.valid = torch.tensor([rt.tokens], dtype=torch.int32, device=gen_dev)
            self.inputs += ["pmap", "probs", "n_used", "inv", "valid"]
        if "unpermute" in groups:
            self.eo = inputs.expert_output_input(rt, PERMUTED["hidden"], seed=seed + 5,
                                                 device=gen_dev)
            self.unp_out = z(w["permuted"]["tokens"], PERMUTED["hidden"])
            self.inputs += ["eo"]
            self.outputs += ["unp_out"]
        if "residual" in groups:
            res = inputs.residual_inputs((w["residual"]["rows"], RESIDUAL["hidden"]),
                                         torch.bfloat16, seed=seed + 6, device=gen_dev)
            self.res_e, self.res_s, self.res_r = (res["expert_output"],
                                                  res["shared_expert_output"], res["residual"])
            self.res_out = z(w["residual"]["rows"], RESIDUAL["hidden"])
            self.inputs += ["res_e", "res_s", "res_r"]
            self.outputs += ["res_out"]
        if "router_weight_fwd" in self.names:
            # chained epilogue: the router-weight forward writes the first rows of the
            # residual's expert output (a tensor of its own when run alone)
            n = self.rw_x.shape[0]
            self.rw_out = self.res_e[:n] if "residual" in groups else z(n, ROUTER["hidden"])
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)
        for k in self.inputs:
            setattr(self, k, getattr(self, k).to(device))

    def kernels(self):
        """(name, launch) pairs, in MoE-layer order."""
        from moe_expert_epilogue_b200 import ops
        L = SWIGLU["limit"]
        P = PERMUTED
        table = {
            "swiglu_fwd": lambda: ops.swiglu_clamped_fwd(self.sw_x, self.sw_p, L, out=self.sw_y),
            "router_weight_fwd": lambda: ops.router_weight_mul_fwd(
                self.rw_x, self.rw_p, torch.bfloat16, out=self.rw_out),
            "act_sqrelu": lambda: ops.act_with_probs_permuted(
                ops.MOE_ACT_SQRELU, self.act_x, self.pmap, self.n_used, self.probs, 1.0, True,
                out=self.act_o1, dev_err=self.dev_err),
            "act_sqrelu_clamp": lambda: ops.act_with_probs_permuted(
                ops.MOE_ACT_SQRELU_CLAMP, self.act_x, self.pmap, self.n_used, self.probs,
                P["scale"], True, out=self.act_o2, dev_err=self.dev_err),
            "act_swiglu": lambda: ops.act_with_probs_permuted(
                ops.MOE_ACT_SWIGLU, self.act_x2, self.pmap, self.n_used, self.probs, 1.0, True,
                out=self.act_o3, dev_err=self.dev_err),
            "unpermute": lambda: ops.unpermute_ordered(self.eo, self.inv, self.valid,
                                                       self.unp_out, dev_err=self.dev_err),
            "residual_add": lambda: ops.residual_add(self.res_e, self.res_s, self.res_r,
                                                     out=self.res_out),
            "router_weight_bwd": lambda: ops.router_weight_mul_bwd(
                self.rw_g, self.rw_x, self.rw_p, grad_x=self.rw_gx, grad_probs=self.rw_gp),
            "swiglu_bwd": lambda: ops.swiglu_clamped_bwd(self.sw_x, self.sw_p, self.sw_gy, L,
                                                         grad_x=self.sw_gx,
                                                         grad_probs=self.sw_gp),
        }
        return [(n, table[n]) for n in self.names]


# ---------------------------------------------------------------- next rows

def time_launches(fn, reps, device):
    """Mean device time (ms) of `reps` back-to-back calls of fn after 3 warm-ups."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize(device)
    return a.elapsed_time(b) / reps


NEXT_ROWS = ("weighted_silu_mul_bounded", "epilogue_fused", "ordered_reduce_scatter_v",
             "unpermute_reduce_scatter", "dtype_variants")
RS_WORLD = 8  # EP ranks of the rank-order reduce-scatter, all blocks on this GPU


def measure_next_rows(device, seed, reps, peak, scale=1.0, only=None):
    """The ops beyond the step: the device-bounded weighted SwiGLU, the fused
    router-weight -> unpermute -> residual chain (against the same chain as
    three launches), the rank-order reduce-scatter, the EP combine and the
    other storage dtypes of the SwiGLU and the router-weight probabilities.
    Timed after the step, outside its timed region."""
    from moe_expert_epilogue_b200 import inputs, ops
    out = {}
    T = scaled(scale)["permuted"]["tokens"]
    K, E, A, H = PERMUTED["top_k"], PERMUTED["experts"], PERMUTED["align"], PERMUTED["hidden"]
    rows, half_n = T * K, PERMUTED["width"]
    if only in (None, "weighted_silu_mul_bounded"):
        out.update(_measure_bounded(device, seed, reps, peak, rows, half_n))
    if only in (None, "epilogue_fused"):
        out.update(_measure_fused(device, seed, reps, peak, T, K, E, A, H))
    if only in (None, "ordered_reduce_scatter_v"):
        out.update(_measure_reduce_scatter(device, seed, reps, peak, T, H))
    if only in (None, "unpermute_reduce_scatter"):
        out.update(_measure_ep_combine(device, seed, reps, peak, T, K, E, A, H,
                                       long_tokens=8192 if scale == 1.0 else None))
    if only in (None, "dtype_variants"):
        out["dtype_variants"] = _measure_dtype_variants(device, seed, reps, peak, scale)
    return out


def _measure_dtype_variants(device, seed, reps, peak, scale=1.0):
    """The other storage dtypes of the hot path's ops: the clamped SwiGLU fwd and
    bwd in fp16 and fp32 at the headline shape, and the router-weight fwd and
    bwd (x saved) with bf16 and fp16 routing probabilities at [16384, 7168]."""
    from moe_expert_epilogue_b200 import ops
    out = {}
    R, I, L = int(SWIGLU["rows"] * scale), SWIGLU["inter"], SWIGLU["limit"]
    g = torch.Generator(device=device).manual_seed(seed + 41)
    for dt, name in ((torch.float16, "fp16"), (torch.float32, "fp32")):
        es = torch.empty((), dtype=dt).element_size()
        x = (torch.randn(R, 2 * I, generator=g, device=device) * SWIGLU["sigma"]).to(dt)
        gy = torch.randn(R, I, generator=g, device=device).to(dt)
        p = torch.rand(R, 1, generator=g, device=device)
        y = torch.empty(R, I, dtype=dt, device=device)
        gx = torch.empty(R, 2 * I, dtype=dt, device=device)
        gp = torch.empty(R, 1, dtype=torch.float32, device=device)
        ms_f = time_launches(lambda: ops.swiglu_clamped_fwd(x, p, L, out=y), reps, device)
        ms_b = time_launches(lambda: ops.swiglu_clamped_bwd(x, p, gy, L, grad_x=gx, grad_probs=gp),
                             reps, device)
        nb_f = R * (2 * I * es + 4 + I * es)
        nb_b = R * (2 * I * es + I * es + 4 + 2 * I * es + 4)
        out[f"swiglu_{name}"] = {"shape": f"rows {R}, inter {I}, L {L}, {name}",
                                 "fwd": _entry(ms_f, nb_f, peak), "bwd": _entry(ms_b, nb_b, peak),
                                 "pair": _entry(ms_f + ms_b, nb_f + nb_b, peak)}
        del x, gy, y, gx
    Rr, H = int(ROUTER["rows"] * scale), ROUTER["hidden"]
    x = torch.randn(Rr, H, generator=g, device=device).to(torch.bfloat16)
    gr = torch.randn(Rr, H, generator=g, device=device).to(torch.bfloat16)
    o = torch.empty_like(x)
    gxr = torch.empty_like(x)
    for pdt, name in ((torch.bfloat16, "bf16"), (torch.float16, "fp16")):
        p = (torch.rand(Rr, 1, generator=g, device=device) + 0.01).to(pdt)
        gpr = torch.empty(Rr, 1, dtype=pdt, device=device)
        ms_f = time_launches(lambda: ops.router_weight_mul_fwd(x, p, torch.bfloat16, out=o), reps,
                             device)
        ms_b = time_launches(lambda: ops.router_weight_mul_bwd(gr, x, p, grad_x=gxr,
                                                               grad_probs=gpr), reps, device)
        nb_f = Rr * (H * 2 * 2 + 2)
        nb_b = Rr * (H * 2 * 3 + 2 + 2)
        out[f"router_weight_probs_{name}"] = {
            "shape": f"[{Rr}, {H}] bf16 x, {name} probs",
            "fwd": _entry(ms_f, nb_f, peak), "bwd_save_x": _entry(ms_b, nb_b, peak)}
    torch.cuda.empty_cache()
    return out


def _graph_time(fn, reps, device):
    """Mean device time of fn replayed as one CUDA graph (fn issues several
    short launches whose host overhead would otherwise show)."""
    fn()
    torch.cuda.synchronize(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    ms = time_launches(graph.replay, reps, device)
    del graph
    return ms


def _measure_ep_combine(device, seed, reps, peak, T, K, E, A, H, world=RS_WORLD,
                        long_tokens=8192):
    """EP combine with every rank's expert rows on this GPU: the fused kernel
    (one launch per rank) against the pages' two steps with the library's own
    kernels (each rank's unpermute into a partial block, then one
    reduce-scatter launch per rank)."""
    from moe_expert_epilogue_b200 import inputs, ops
    case = inputs.ep_combine_inputs(world, T, K, E // world, A, H, seed=seed + 9, device=device)
    eo_t = ops.pointer_table(case.expert_outputs)
    inv_t = ops.pointer_table(case.inverse_maps)
    offs = case.rank_token_offset
    ep = torch.tensor([T], dtype=torch.int32, device=device)
    outs = [torch.empty(c, H, dtype=torch.bfloat16, device=device) for c in case.counts]

    def fused():
        for r in range(world):
            ops.unpermute_reduce_scatter(eo_t, torch.bfloat16, case.max_rows, inv_t, E // world, T,
                                         ep, r, offs, H, out=outs[r])
    blocks = [torch.empty(T, H, dtype=torch.bfloat16, device=device) for _ in range(world)]
    blk_t = ops.pointer_table(blocks)

    def two_step():
        for q in range(world):
            ops.unpermute_ordered(case.expert_outputs[q], case.inverse_maps[q], ep, blocks[q])
        for r in range(world):
            ops.ordered_reduce_scatter_v(blk_t, r, offs, ep, T, H, torch.bfloat16, out=outs[r])
    ms_f = _graph_time(fused, reps, device)
    ms_2 = _graph_time(two_step, reps, device)
    live = T * K
    nb_f = live * H * 2 + world * T * (E // world) * 4 + T * H * 2
    nb_2 = (live * H * 2 + world * T * (E // world) * 4 + world * T * H * 2) \
        + (world * T * H * 2 + T * H * 2)
    res = {
        "shape": f"{world} ranks x {E // world} experts, {T} tokens top-{K}, hidden {H}, bf16, "
                 f"all ranks' expert rows on one GPU, one launch per rank",
        "us": round(ms_f * 1e3, 2), "bytes": nb_f, "gbs": round(nb_f / ms_f / 1e6, 1),
        "frac": round(nb_f / ms_f / 1e6 / peak, 4),
        "two_step_us": round(ms_2 * 1e3, 2), "two_step_bytes": nb_2,
        "speedup_vs_two_step": round(ms_2 / ms_f, 3)}
    del case, eo_t, inv_t, outs, blocks, blk_t
    torch.cuda.empty_cache()
    if long_tokens:                       # longer launches: long_tokens tokens a rank
        TL = long_tokens * world
        case = inputs.ep_combine_inputs(world, TL, K, E // world, A, H, seed=seed + 10,
                                        device=device)
        eo_t = ops.pointer_table(case.expert_outputs)
        inv_t = ops.pointer_table(case.inverse_maps)
        ep = torch.tensor([TL], dtype=torch.int32, device=device)
        outs = [torch.empty(c, H, dtype=torch.bfloat16, device=device) for c in case.counts]

        def fused_long():
            for r in range(world):
                ops.unpermute_reduce_scatter(eo_t, torch.bfloat16, case.max_rows, inv_t,
                                             E // world, TL, ep, r, case.rank_token_offset, H,
                                             out=outs[r])
        ms = _graph_time(fused_long, max(3, reps // 4), device)
        nb = TL * K * H * 2 + world * TL * (E // world) * 4 + TL * H * 2
        res["long"] = {"shape": f"{TL} tokens ({long_tokens} a rank), otherwise as above",
                       "us": round(ms * 1e3, 2), "bytes": nb, "gbs": round(nb / ms / 1e6, 1),
                       "frac": round(nb / ms / 1e6 / peak, 4)}
        del case, eo_t, inv_t, outs
        torch.cuda.empty_cache()
    return {"unpermute_reduce_scatter": res}


def _measure_reduce_scatter(device, seed, reps, peak, T, H, world=RS_WORLD):
    """The rank-order reduce-scatter with every EP rank's [T, H] block on this
    GPU: one pass = the world's launches (one per rank) back to back, together
    reading every block once and writing T rows.  On several GPUs the same
    kernel reads (world-1)/world of these bytes over NVLink instead."""
    from moe_expert_epilogue_b200 import inputs, ops
    case = inputs.reduce_scatter_inputs(world, T, H, seed=seed + 8, device=device)
    table = ops.pointer_table(case.buffers)
    offs = case.rank_token_offset
    ep = torch.tensor([case.ep_tokens], dtype=torch.int32, device=device)
    outs = [torch.empty(c, H, dtype=torch.bfloat16, device=device) for c in case.counts]

    def one_pass():
        for r in range(world):
            ops.ordered_reduce_scatter_v(table, r, offs, ep, T, H, torch.bfloat16, out=outs[r])
    # each launch is ~10 us of device time: replay the pass as a CUDA graph so
    # that host launch overhead does not show in the device time
    ms = _graph_time(one_pass, reps, device)
    nb = world * T * H * 2 + T * H * 2
    return {"ordered_reduce_scatter_v": {
        "shape": f"{world} ranks' bf16 blocks of {T} tokens x hidden {H} on one GPU, "
                 f"{world} launches (ragged per-rank rows)",
        "us": round(ms * 1e3, 2), "bytes": nb, "gbs": round(nb / ms / 1e6, 1),
        "frac": round(nb / ms / 1e6 / peak, 4)}}


def _measure_bounded(device, seed, reps, peak, rows, half_n):
    from moe_expert_epilogue_b200 import ops
    out = {}
    g = torch.Generator(device=device).manual_seed(seed + 7)
    y = (torch.randn(rows, 2 * half_n, generator=g, device=device) * 3).to(torch.bfloat16)
    w = torch.rand(rows, generator=g, device=device)
    bound = torch.tensor([rows * half_n], dtype=torch.int64, device=device)
    o = torch.empty(rows, half_n, dtype=torch.bfloat16, device=device)
    ms = time_launches(lambda: ops.weighted_silu_mul_bounded(y, w, bound, out=o), reps, device)
    nb = rows * (2 * half_n * 2 + 4 + half_n * 2)
    out["weighted_silu_mul_bounded"] = {
        "shape": f"rows {rows} (all live), half_n {half_n}", "us": round(ms * 1e3, 2),
        "bytes": nb, "gbs": round(nb / ms / 1e6, 1), "frac": round(nb / ms / 1e6 / peak, 4)}
    return out


def _measure_fused(device, seed, reps, peak, T, K, E, A, H):
    from moe_expert_epilogue_b200 import inputs, ops
    out = {}
    rt = inputs.routing(T, K, E, A, seed=seed + 2, device=device)
    eo = inputs.expert_output_input(rt, H, seed=seed + 5, device=device)
    pm = rt.permutation_map
    rp = torch.where(pm >= 0, rt.probs[pm.clamp(min=0).long()],
                     torch.zeros((), device=device)).float()
    res = inputs.residual_inputs((T, H), torch.bfloat16, seed=seed + 6, device=device)
    sh, rs = res["shared_expert_output"], res["residual"]
    vt = torch.tensor([T], dtype=torch.int32, device=device)
    fo = torch.empty_like(rs)
    ms_f = time_launches(lambda: ops.epilogue_fused(eo, rp, rt.inverse_map, vt, sh, rs, out=fo),
                         reps, device)
    wbuf, routed, co = torch.empty_like(eo), torch.empty_like(rs), torch.empty_like(rs)

    def chained():
        ops.router_weight_mul_fwd(eo, rp, torch.bfloat16, out=wbuf)
        ops.unpermute_ordered(wbuf, rt.inverse_map, vt, routed)
        ops.residual_add(routed, sh, rs, out=co)
    ms_c = time_launches(chained, reps, device)
    live = T * K
    nb_f = live * H * 2 + live * 4 + T * E * 4 + 3 * T * H * 2
    nb_c = (rt.max_rows * H * 2 * 2 + rt.max_rows * 4) + (live * H * 2 + T * E * 4 + T * H * 2) \
        + 4 * T * H * 2
    out["epilogue_fused"] = {
        "shape": f"{T} tokens x top-{K} of {E}, hidden {H}, bf16", "us": round(ms_f * 1e3, 2),
        "bytes": nb_f, "gbs": round(nb_f / ms_f / 1e6, 1), "frac": round(nb_f / ms_f / 1e6 / peak, 4),
        "chained_three_launches_us": round(ms_c * 1e3, 2), "chained_bytes": nb_c,
        "speedup_vs_chained": round(ms_c / ms_f, 3)}
    return out


# ---------------------------------------------------------------- configurations

CONFIG_ROWS = ("swiglu_small", "router_weight_variants", "residual_add_variants",
               "unpermute_fp32_out")
L2_FLUSH_BYTES = 256 << 20   # twice the 126 MB L2


def _entry(ms, nbytes, peak, **extra):
    gbs = nbytes / (ms * 1e-3) / 1e9
    return dict(us=round(ms * 1e3, 2), bytes=nbytes, gbs=round(gbs, 1),
                frac=round(gbs / peak, 4), **extra)


def measure_configs(device, seed, reps, peak, only=None):
    """The workload's configurations the step does not run, each timed alone
    after the step (outside its timed region): the small SwiGLU (latency-bound,
    L2 flushed before every pair), the router-weight multiply with fp32 output
    and with and without saved x, the residual add in bf16 / fp16 / fp32 alone
    and chained after the router-weight forward of the same output dtype, and
    the unpermute into fp32.  Inputs larger than L2 except the small SwiGLU."""
    out = {}
    if only in (None, "swiglu_small"):
        out["swiglu_small"] = _measure_swiglu_small(device, seed, max(reps, 50), peak)
    if only in (None, "router_weight_variants"):
        out["router_weight_variants"] = _measure_router_variants(device, seed, reps, peak)
    if only in (None, "residual_add_variants"):
        out["residual_add_variants"] = _measure_residual_variants(device, seed, reps, peak)
    if only in (None, "unpermute_fp32_out"):
        out["unpermute_fp32_out"] = _measure_unpermute_fp32(device, seed, reps, peak)
    torch.cuda.empty_cache()
    return out


def _measure_swiglu_small(device, seed, reps, peak):
    """rows 256, inter 512 (x ~N(0, 2^2), probs ~U(0,1)), L = 7 and inf: per
    launch with the L2 flushed before every fwd/bwd pair (cold), and replayed
    as a CUDA graph with the 1 MB working set in L2 (hot)."""
    from moe_expert_epilogue_b200 import inputs, ops
    R, I = 256, 512
    d = inputs.swiglu_inputs(R, I, sigma=2.0, seed=seed, device=device)
    x, p, gy = d["x"], d["probs"], d["grad_y"]
    y, gx = torch.empty(R, I, dtype=torch.bfloat16, device=device), torch.empty_like(x)
    gp = torch.empty(R, 1, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    nb_f, nb_b = R * (6 * I + 4), R * (10 * I + 8)
    res = {"shape": f"rows {R}, inter {I}, bf16; latency-bound (the working set fits in L2)"}
    for L in (7.0, float("inf")):
        fwd = lambda: ops.swiglu_clamped_fwd(x, p, L, out=y)  # noqa: E731
        bwd = lambda: ops.swiglu_clamped_bwd(x, p, gy, L, grad_x=gx, grad_probs=gp)  # noqa: E731
        for _ in range(3):
            fwd()
            bwd()
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(reps)]
        for e in evs:
            flush.zero_()
            e[0].record()
            fwd()
            e[1].record()
            bwd()
            e[2].record()
        torch.cuda.synchronize(device)
        tf = sorted(e[0].elapsed_time(e[1]) for e in evs)[reps // 2]
        tb = sorted(e[1].elapsed_time(e[2]) for e in evs)[reps // 2]
        hot_f = _graph_time(fwd, reps, device)      # one launch is shorter than its host call
        hot_b = _graph_time(bwd, reps, device)
        key = "L7" if L == 7.0 else "Linf"
        res[key] = {"fwd_cold": _entry(tf, nb_f, peak, rows_per_s=R / (tf * 1e-3)),
                    "bwd_cold": _entry(tb, nb_b, peak, rows_per_s=R / (tb * 1e-3)),
                    "fwd_hot_us": round(hot_f * 1e3, 2), "bwd_hot_us": round(hot_b * 1e3, 2),
                    "timing": f"median of {reps} flushed launches; hot = mean of {reps} "
                              "graph replays of one launch (working set in L2)"}
    return res


def _measure_router_variants(device, seed, reps, peak):
    """[16384, 7168] bf16 x, U(0.01, 1) probs: the forward into bf16 and fp32,
    the backward from a bf16 and an fp32 gradient, with x saved (grad_probs
    computed) and without (x not read)."""
    from moe_expert_epilogue_b200 import inputs, ops
    Rr, H = ROUTER["rows"], ROUTER["hidden"]
    d = inputs.router_weight_inputs(Rr, H, seed=seed + 1, device=device)
    x, p, g16 = d["x"], d["probs"], d["grad_out"]
    g32 = g16.float()
    n = Rr * H
    o16 = torch.empty(Rr, H, dtype=torch.bfloat16, device=device)
    o32 = torch.empty(Rr, H, dtype=torch.float32, device=device)
    gx = torch.empty(Rr, H, dtype=torch.bfloat16, device=device)
    gp = torch.empty(Rr, 1, device=device)
    res = {"shape": f"[{Rr}, {H}] bf16 x, fp32 probs"}
    runs = {
        "fwd_out_bf16": (lambda: ops.router_weight_mul_fwd(x, p, out=o16), n * 4 + Rr * 4),
        "fwd_out_fp32": (lambda: ops.router_weight_mul_fwd(x, p, out=o32), n * 6 + Rr * 4),
        "bwd_g_bf16_save_x": (lambda: ops.router_weight_mul_bwd(g16, x, p, grad_x=gx,
                                                                grad_probs=gp), n * 6 + Rr * 8),
        "bwd_g_bf16_no_x": (lambda: ops.router_weight_mul_bwd(g16, None, p, torch.bfloat16,
                                                              grad_x=gx), n * 4 + Rr * 4),
        "bwd_g_fp32_save_x": (lambda: ops.router_weight_mul_bwd(g32, x, p, grad_x=gx,
                                                                grad_probs=gp), n * 8 + Rr * 8),
        "bwd_g_fp32_no_x": (lambda: ops.router_weight_mul_bwd(g32, None, p, torch.bfloat16,
                                                              grad_x=gx), n * 6 + Rr * 4),
    }
    for name, (fn, nb) in runs.items():
        ms = time_launches(fn, reps, device)
        res[name] = _entry(ms, nb, peak, rows_per_s=Rr / (ms * 1e-3))
    return res


def _measure_residual_variants(device, seed, reps, peak):
    """[32768, 7168] N(0,1) in bf16, fp16 and fp32: the residual add alone, and
    chained after the router-weight forward that produces its expert output
    (bf16 x of the same shape, U(0.01, 1) probs, output in the add's dtype) on
    one stream as one epilogue pass."""
    from moe_expert_epilogue_b200 import inputs, ops
    R, H = RESIDUAL["rows"], RESIDUAL["hidden"]
    n = R * H
    rw = inputs.router_weight_inputs(R, H, seed=seed + 6, device=device)
    x, p = rw["x"], rw["probs"]
    del rw
    res = {"shape": f"[{R}, {H}]"}
    for dt, name in ((torch.bfloat16, "bf16"), (torch.float16, "fp16"), (torch.float32, "fp32")):
        t = inputs.residual_inputs((R, H), dt, seed=seed + 6, device=device)
        e, s, r = t["expert_output"], t["shared_expert_output"], t["residual"]
        o = torch.empty_like(r)
        es = o.element_size()
        ms = time_launches(lambda: ops.residual_add(e, s, r, out=o), reps, device)
        res[name] = _entry(ms, 4 * n * es, peak, rows_per_s=R / (ms * 1e-3))

        def chain():
            ops.router_weight_mul_fwd(x, p, out=e)
            ops.residual_add(e, s, r, out=o)
        ms = time_launches(chain, reps, device)
        nb = (n * 2 + n * es + R * 4) + 4 * n * es
        res[name + "_chained"] = _entry(ms, nb, peak, rows_per_s=R / (ms * 1e-3))
        del t, e, s, r, o
        torch.cuda.empty_cache()
    return res


def _measure_unpermute_fp32(device, seed, reps, peak):
    """The fixed-order unpermute of the step's routing (8192 tokens, top-8 of
    64, hidden 4096, bf16 expert rows) into an fp32 output."""
    from moe_expert_epilogue_b200 import inputs, ops
    P = PERMUTED
    rt = inputs.routing(P["tokens"], P["top_k"], P["experts"], P["align"], seed=seed + 2,
                        device=device)
    eo = inputs.expert_output_input(rt, P["hidden"], seed=seed + 5, device=device)
    valid = torch.tensor([rt.tokens], dtype=torch.int32, device=device)
    o = torch.empty(rt.tokens, P["hidden"], dtype=torch.float32, device=device)
    ms = time_launches(lambda: ops.unpermute_ordered(eo, rt.inverse_map, valid, o), reps, device)
    live = rt.tokens * rt.top_k
    nb = live * P["hidden"] * 2 + rt.tokens * P["experts"] * 4 + rt.tokens * P["hidden"] * 4
    return _entry(ms, nb, peak, rows_per_s=rt.tokens / (ms * 1e-3),
                  shape=f"{rt.tokens} tokens x top-{rt.top_k} of {P['experts']}, hidden "
                        f"{P['hidden']}, bf16 -> fp32")


# ---------------------------------------------------------------- collectives (N > 1)

PEER_GBS = 770.0   # measured peer copy on this node type, per direction per GPU


class _Clock:
    """CUDA events on the current stream (host clock on a CPU process group)."""

    def __init__(self, device):
        self.cuda = device.type == "cuda"
        self.device = device

    def mark(self):
        if self.cuda:
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            return e
        return time.perf_counter()

    def ms(self, a, b):
        if self.cuda:
            torch.cuda.synchronize(self.device)
            return a.elapsed_time(b)
        return (b - a) * 1e3


def measure_collectives(device, seed, reps, tokens=8192, hidden=4096, top_k=8,
                        experts_per_rank=8, backend=None, return_outputs=False):
    """The exchange steps across the ranks of the process group (one per GPU),
    timed after the step: the rank-order reduce-scatter (every rank's block of
    bf16 partials for all `tokens` token rows in a symmetric buffer) and the EP
    combine (every rank's expert rows and inverse map in two symmetric
    buffers), both through `symmetric` -- peer buffers read over NVLink with
    plain loads.  Per collective: the kernel alone (CUDA events around the
    launch, between the two stream barriers; max over ranks) and the whole
    call (barriers included); NVLink bytes are the rows this rank reads from
    its peers.  `backend` replaces the CUDA IPC mapping (CPU tests)."""
    import torch.distributed as dist
    from moe_expert_epilogue_b200 import inputs, symmetric
    rank, world = dist.get_rank(), dist.get_world_size()
    clock = _Clock(device)
    out, outputs = {"world": world}, {}
    peak_hbm, _ = hbm_peak()
    dt, H = torch.bfloat16, hidden

    def run(call):
        """call(hooks) runs one collective; hooks = (before, after) run around
        its launch.  Returns the mean kernel and whole-call ms, max over ranks."""
        for _ in range(2):
            call(None)
        kern, whole = [], []
        for _ in range(reps):
            marks = []
            hook = lambda: marks.append(clock.mark())  # noqa: E731
            a = clock.mark()
            call((hook, hook))
            b = clock.mark()
            kern.append(clock.ms(marks[0], marks[1]))
            whole.append(clock.ms(a, b))
        return (max_over_ranks(sum(kern) / reps, device),
                max_over_ranks(sum(whole) / reps, device))

    def entry(k_ms, w_ms, local_bytes, remote_bytes, **extra):
        t_link = remote_bytes / (PEER_GBS * 1e9) * 1e3
        t_hbm = local_bytes / (peak_hbm * 1e9) * 1e3
        return dict(kernel_us=round(k_ms * 1e3, 2), call_us=round(w_ms * 1e3, 2),
                    bytes_read_written=local_bytes, nvlink_bytes=remote_bytes,
                    nvlink_gbs=round(remote_bytes / (k_ms * 1e-3) / 1e9, 1),
                    frac=round(max(t_link, t_hbm) / k_ms, 4),
                    roofline=f"max(NVLink bytes / {PEER_GBS:g} GB/s measured peer copy, "
                             f"bytes / {peak_hbm:g} GB/s HBM) / kernel time", **extra)

    # rank-order reduce-scatter
    case = inputs.reduce_scatter_inputs(world, tokens, H, seed=seed + 8, device=device)
    cap, mine = tokens, case.counts[rank]
    symm = symmetric.SymmetricBuffer(cap * H * 2, device=device, backend=backend)
    symm.view(dt, (cap, H)).copy_(case.buffers[rank])
    offs, ep = case.rank_token_offset, torch.tensor([case.ep_tokens], dtype=torch.int32,
                                                    device=device)
    rs_out = torch.empty(mine, H, dtype=dt, device=device)
    del case

    k, w = run(lambda hooks: symmetric.ordered_reduce_scatter_v(
        rs_out, symm, offs, ep, cap, H, dt, launch_hooks=hooks))
    out["ordered_reduce_scatter_v"] = entry(
        k, w, mine * H * 2 * (world + 1), mine * H * 2 * (world - 1),
        shape=f"{world} ranks, {tokens} token rows x hidden {H} bf16 partials per rank, "
              f"{mine} rows on this rank")
    if return_outputs:
        outputs["ordered_reduce_scatter_v"] = rs_out.clone()
    symm.close()
    del rs_out

    # EP combine
    ec = inputs.ep_combine_inputs(world, tokens, top_k, experts_per_rank, 128, H,
                                  seed=seed + 9, device=device)
    mine, first = ec.counts[rank], int(ec.rank_token_offset[rank])
    experts = symmetric.SymmetricBuffer(ec.max_rows * H * 2, device=device, backend=backend)
    maps = symmetric.SymmetricBuffer(tokens * experts_per_rank * 4, device=device,
                                     backend=backend)
    experts.view(dt, (ec.max_rows, H)).copy_(ec.expert_outputs[rank])
    maps.view(torch.int32, (tokens, experts_per_rank)).copy_(ec.inverse_maps[rank])
    rows_from = [int((m[first:first + mine] >= 0).sum()) for m in ec.inverse_maps]
    remote_rows = sum(r for q, r in enumerate(rows_from) if q != rank)
    ep_t = torch.tensor([tokens], dtype=torch.int32, device=device)
    offs = ec.rank_token_offset
    ec_out = torch.empty(mine, H, dtype=dt, device=device)
    max_rows = ec.max_rows
    del ec

    k, w = run(lambda hooks: symmetric.unpermute_reduce_scatter(
        ec_out, experts, maps, dt, max_rows, H, experts_per_rank, tokens, offs, ep_t,
        launch_hooks=hooks))
    meta = mine * experts_per_rank * 4
    out["unpermute_reduce_scatter"] = entry(
        k, w, sum(rows_from) * H * 2 + world * meta + mine * H * 2,
        remote_rows * H * 2 + (world - 1) * meta,
        shape=f"{world} ranks x {experts_per_rank} experts, {tokens} tokens top-{top_k}, "
              f"hidden {H} bf16, {mine} tokens on this rank")
    if return_outputs:
        outputs["unpermute_reduce_scatter"] = ec_out.clone()
    experts.close()
    maps.close()
    if device.type != "cuda":
        out["note"] = "CPU process group: protocol check only, times are not GPU times"
    return (out, outputs) if return_outputs else out


# ---------------------------------------------------------------- distributed

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def max_over_ranks(value: float, device) -> float:
    """Max of a scalar over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate_value(bytes_per_step: int, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return bytes_per_step * steps * world / max_seconds / 1e9


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        self.path = tempfile.mktemp(suffix=".csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 5 and os.path.getsize(self.path) == 0:
                time.sleep(0.02)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            self.proc.wait(timeout=5)

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]),
                                 power=float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                                 active=parts[4], hw=parts[5], hwt=parts[6], swt=parts[7],
                                 pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] > 250.0] or rows
        sms = sorted(r["sm"] for r in loaded)
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": sms[len(sms) // 2], "sm_max_mhz": loaded[0]["max"],
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------- peaks, traffic

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def source_digest(fn: str) -> str:
    csrc = os.path.join(ROOT, "moe_expert_epilogue_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted([fn, "common.cuh"]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            entry = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if entry.get("source_digest") != source_digest(KERNEL_SOURCES[kernel]):
        return None
    return entry.get("bytes_per_launch")


# ---------------------------------------------------------------- our arm

def _kernel_stats(times_ms, nbytes, rows, peak):
    """Mean / median of one kernel's event durations and its GB/s."""
    times = sorted(times_ms)
    avg_ms = sum(times) / len(times)
    gbs = nbytes / (avg_ms * 1e-3) / 1e9
    st = {"us": round(avg_ms * 1e3, 2), "median_us": round(times[len(times) // 2] * 1e3, 2),
          "bytes": nbytes, "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
          "launches_timed": len(times), "share": None}
    if rows:
        st["rows_per_s"] = rows / (avg_ms * 1e-3)
    return st


def run_ours(args):
    from moe_expert_epilogue_b200 import build as mbuild
    rank, local_rank, world = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device,
                                timeout=datetime.timedelta(seconds=120))
    if not mbuild.up_to_date():
        if rank == 0:
            mbuild.build()
        barrier(device)

    only = set(args.kernel.split(",")) if args.kernel else None
    if only and len(only) == 1 and next(iter(only)) in NEXT_ROWS + CONFIG_ROWS:
        # a next-row op or a configuration alone (profiling captures)
        peak, _ = hbm_peak()
        name = next(iter(only))
        if name in NEXT_ROWS:
            res = measure_next_rows(device, 1000 * rank, args.steps, peak, args.scale, only=name)
        else:
            res = measure_configs(device, 1000 * rank, args.steps, peak, only=name)
        if rank == 0:
            print(json.dumps({"kernel": args.kernel, "scale": args.scale, "result": res}),
                  flush=True)
        return
    if only and not only <= set(ORDER):
        raise SystemExit(f"unknown --kernel {args.kernel}; choose from "
                         f"{ORDER + list(NEXT_ROWS) + list(CONFIG_ROWS)}")
    batch = Batch(device, seed=1000 * rank, scale=args.scale, kernels=only)
    kernels = batch.kernels()
    nbytes = algorithmic_bytes(batch.rt.n_used, args.scale)
    nbytes = {n: nbytes[n] for n, _ in kernels}
    rows = rows_per_launch(args.scale)
    bytes_per_step = sum(nbytes.values())
    stream = torch.cuda.current_stream(device)
    head = all(h in nbytes for h in HEAD)

    for _ in range(args.warmup):
        for _, fn in kernels:
            fn()
    torch.cuda.synchronize(device)

    K = args.steps
    every = max(1, args.event_every)
    probed = [k for k in range(K) if k % every == every - 1] or [K - 1]
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    # the SwiGLU pair: events before the forward, between the two, after the backward
    hev = [(mk(), mk(), mk()) for _ in range(K)] if head else None
    ev = {name: {k: (mk(), mk()) for k in probed} for name, _ in kernels if name not in HEAD
          or not head}
    t_start, t_end = mk(), mk()
    sampler = ClockSampler(device.index) if not args.no_clocks else contextlib.nullcontext()
    with sampler:
        barrier(device)
        torch.cuda.synchronize(device)
        t_start.record(stream)
        for k in range(K):
            probe = k in probed
            for name, fn in kernels:
                if head and name == HEAD[0]:
                    hev[k][0].record(stream)
                    fn()
                    hev[k][1].record(stream)
                elif head and name == HEAD[1]:
                    fn()
                    hev[k][2].record(stream)
                elif probe:
                    ev[name][k][0].record(stream)
                    fn()
                    ev[name][k][1].record(stream)
                else:
                    fn()
        t_end.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
    step_ms = t_start.elapsed_time(t_end)
    max_step_ms = max_over_ranks(step_ms, device)
    clocks = sampler.summary() if not args.no_clocks else None

    per_kernel = {}
    peak, peak_kind = hbm_peak()
    for name, _ in kernels:
        if head and name in HEAD:
            i = HEAD.index(name)
            times = [e[i].elapsed_time(e[i + 1]) for e in hev]
        else:
            times = [a.elapsed_time(b) for a, b in ev[name].values()]
        per_kernel[name] = _kernel_stats(times, nbytes[name], rows[name], peak)
    total_kernel_ms = sum(v["us"] for v in per_kernel.values())
    for v in per_kernel.values():
        v["share"] = round(v["us"] / total_kernel_ms, 4)

    # the headline: the SwiGLU pair over all K steps (else, for a --kernel
    # subset without it, the selected kernels' whole steps)
    if head:
        head_bytes = nbytes[HEAD[0]] + nbytes[HEAD[1]]
        head_ms = sum(e[0].elapsed_time(e[2]) for e in hev)
    else:
        head_bytes, head_ms = bytes_per_step, step_ms
    max_head_ms = max_over_ranks(head_ms, device)
    value = aggregate_value(head_bytes, K, world, max_head_ms * 1e-3)
    dom_set = HEAD if head else list(per_kernel)
    dominant = max(dom_set, key=lambda n: per_kernel[n]["us"])
    d = per_kernel[dominant]
    step_dom = max(per_kernel, key=lambda n: per_kernel[n]["us"])
    sd = per_kernel[step_dom]
    sw = None
    if head:
        us = max_head_ms * 1e3 / K
        sw = {"us_per_step": round(us, 2), "bytes": head_bytes,
              "gbs": round(head_bytes / (us * 1e-6) / 1e9, 1),
              "frac": round(head_bytes / (us * 1e-6) / 1e9 / peak, 4),
              "rows_per_s": rows[HEAD[0]] / (us * 1e-6),
              "fwd_frac": per_kernel[HEAD[0]]["frac"], "bwd_frac": per_kernel[HEAD[1]]["frac"],
              "steps_timed": K}

    e2e = e2e_step = None
    if not args.no_e2e and not args.kernel:
        e2e_step = run_e2e(args, device, 1000 * rank, first=batch)
        if head:
            e2e = run_e2e(args, device, 1000 * rank + 11, names=HEAD)
    n_used, n_kernels = batch.rt.n_used, len(kernels)
    next_rows = configs = collectives = None
    if not args.kernel:
        del batch, kernels
        torch.cuda.empty_cache()
        if not args.no_configs:
            configs = measure_configs(device, 1000 * rank, 20, peak)
        if not args.no_next_rows:
            next_rows = measure_next_rows(device, 1000 * rank, 20, peak)
        if world > 1 and not args.no_collectives:
            try:
                collectives = measure_collectives(device, 1000, 20)
            except Exception as e:  # the step's numbers still print; the failure is reported
                collectives = {"error": f"{type(e).__name__}: {e}"[:300]}

    if args.kernel or args.scale != 1.0:
        workload = f"{args.kernel or 'all'} at scale {args.scale:g} of: {WORKLOAD_NAME}"
    else:
        workload = HEADLINE_NAME
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(max_head_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload, "bytes_per_step": head_bytes,
                   "timed_in": "every step of the pass: " + WORKLOAD_NAME,
                   "l2": "no flush: every kernel streams > 126 MB (inputs larger than L2)",
                   "parallelism": f"weak: {world} independent replica(s), one per GPU",
                   "per_kernel_events": f"SwiGLU fwd / bwd on all {K} timed steps; the other "
                                        f"kernels on {len(probed)} of them (every {every}th)",
                   "n_used": n_used},
        "swiglu_fwd_bwd": sw,
        "roofline": {"kernel": dominant, "bound": "hbm", "achieved": d["gbs"], "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": d["frac"],
                     "algorithmic_bytes": d["bytes"],
                     "traffic": ncu_traffic(dominant) if args.scale == 1.0 else None,
                     "region": ({"kernels": list(HEAD), "achieved": sw["gbs"],
                                 "frac": sw["frac"], "algorithmic_bytes": head_bytes}
                                if sw else None)},
        "step": {"ms": round(max_step_ms / K, 4), "bytes": bytes_per_step,
                 "gbs": round(aggregate_value(bytes_per_step, K, world, max_step_ms * 1e-3), 1),
                 "frac": round(aggregate_value(bytes_per_step, K, 1, max_step_ms * 1e-3) / peak, 4),
                 "kernels": n_kernels, "e2e": e2e_step,
                 "roofline": {"kernel": step_dom, "achieved": sd["gbs"], "frac": sd["frac"],
                              "algorithmic_bytes": sd["bytes"],
                              "traffic": ncu_traffic(step_dom) if args.scale == 1.0 else None}},
        "kernels": per_kernel,
        "gpu_launches": K * n_kernels,
        "clocks": clocks,
        "e2e": e2e,
        "configs": configs,
        "next_rows": next_rows,
    }
    if collectives is not None:
        line["collectives"] = collectives
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.kernel:
        # about 12 s of one core: every SwiGLU row, 3 passes (~4 s a pass)
        line["cpu_baseline"] = cpu_baseline(args.cpu_sample or 1.0, steps=3)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(args, device, seed, names=None, first=None):
    """The step's kernels `names` (default: all) through the public API with
    inputs in pinned host memory: every step copies all of their inputs host
    -> device, runs the kernels and copies all of their outputs device -> host,
    all inside the timed region.  Steps are pipelined as a user would drive
    them: two device buffer sets (`first`, if given, is one of them), a copy-in
    stream, the compute stream and a copy-out stream, so step k's kernels
    overlap step k+1's inputs and step k-1's outputs on the host link.  Events
    order every reuse of a buffer set."""
    sets = [first or Batch(device, seed=seed, scale=args.scale, kernels=names),
            Batch(device, seed=seed + 7, scale=args.scale, kernels=names)]
    batch = sets[0]
    kernel_sets = [b.kernels() for b in sets]
    nb = algorithmic_bytes(batch.rt.n_used, args.scale)
    step_bytes = sum(nb[n] for n, _ in kernel_sets[0])
    host_in = {k: torch.empty_like(getattr(batch, k), device="cpu").pin_memory()
               for k in batch.inputs}
    for k, h in host_in.items():
        h.copy_(getattr(batch, k))
    host_out = {k: torch.empty_like(getattr(batch, k), device="cpu").pin_memory()
                for k in batch.outputs}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    s_cmp = torch.cuda.current_stream(device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {name: [torch.cuda.Event(), torch.cuda.Event()] for name in ("in", "cmp", "out")}
    for i in range(2):                     # every buffer set starts free
        ev["cmp"][i].record(s_cmp)
        ev["out"][i].record(s_cmp)

    def step(k):
        i, b = k % 2, sets[k % 2]
        s_in.wait_event(ev["cmp"][i])      # step k-2's kernels are done with set i's inputs
        with torch.cuda.stream(s_in):
            for name, h in host_in.items():
                getattr(b, name).copy_(h, non_blocking=True)
        ev["in"][i].record(s_in)
        s_cmp.wait_event(ev["in"][i])
        s_cmp.wait_event(ev["out"][i])     # step k-2's outputs of set i have left
        with torch.cuda.stream(s_cmp):
            for _, fn in kernel_sets[i]:
                fn()
        ev["cmp"][i].record(s_cmp)
        s_out.wait_event(ev["cmp"][i])
        with torch.cuda.stream(s_out):
            for name, h in host_out.items():
                h.copy_(getattr(b, name), non_blocking=True)
        ev["out"][i].record(s_out)

    for k in range(2):
        step(k)
    torch.cuda.synchronize(device)
    n = args.e2e_steps
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    a.record(s_in)
    for k in range(n):
        step(k)
    z.record(s_out)
    torch.cuda.synchronize(device)
    barrier(device)
    ms = max_over_ranks(a.elapsed_time(z), device)
    _, _, world = dist_env()
    return {"value": round(aggregate_value(step_bytes, n, world, ms * 1e-3), 2),
            "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "ms_per_step": round(ms / n, 3),
            "kernels": [name for name, _ in kernel_sets[0]],
            "pipeline": "2 device buffer sets; copy-in, compute and copy-out streams"}


# ---------------------------------------------------------------- CPU oracle

def cpu_sample_workload(frac: float, seed: int = 0, whole_pass: bool = False):
    """A bounded sample of the same workload on the host, same distributions:
    the first `frac` of the SwiGLU rows (the headline), or with `whole_pass`
    the first `frac` of the rows (tokens) of every op of the step."""
    from moe_expert_epilogue_b200 import inputs
    R = max(8, int(SWIGLU["rows"] * frac) // 8 * 8)
    sw = inputs.swiglu_inputs(R, SWIGLU["inter"], sigma=SWIGLU["sigma"], probs="topk_softmax",
                              seed=seed)
    w = dict(R=R, sw=sw, whole_pass=whole_pass)
    if not whole_pass:
        return w
    Rr = max(1, int(ROUTER["rows"] * frac))
    T = max(8, int(PERMUTED["tokens"] * frac))
    Rs = max(1, int(RESIDUAL["rows"] * frac))
    rw = inputs.router_weight_inputs(Rr, ROUTER["hidden"], seed=seed + 1)
    rt = inputs.routing(T, PERMUTED["top_k"], PERMUTED["experts"], PERMUTED["align"], seed=seed + 2)
    ax = inputs.permuted_activation_input(rt, PERMUTED["width"], swiglu=False, seed=seed + 3)
    ax2 = inputs.permuted_activation_input(rt, PERMUTED["width"], swiglu=True, seed=seed + 4)
    eo = inputs.expert_output_input(rt, PERMUTED["hidden"], seed=seed + 5)
    res = inputs.residual_inputs((Rs, RESIDUAL["hidden"]), torch.bfloat16, seed=seed + 6)
    w.update(Rr=Rr, T=T, Rs=Rs, rw=rw, rt=rt, ax=ax, ax2=ax2, eo=eo, res=res)
    return w


def oracle_step(w):
    """One pass of the oracle over the sampled workload (the SwiGLU fwd + bwd,
    or every op of the step); returns its algorithmic bytes."""
    import numpy as np
    import oracle
    from moe_expert_epilogue_b200.inputs import bits
    L, I, W, Hu = SWIGLU["limit"], SWIGLU["inter"], PERMUTED["width"], PERMUTED["hidden"]
    sw, R = w["sw"], w["R"]
    xb, pb, gb = bits(sw["x"]), bits(sw["probs"]), bits(sw["grad_y"])
    oracle.swiglu_clamped_fwd(xb, pb, L)
    nbytes = R * (2 * I * 2 + 4 + I * 2) + R * (2 * I * 2 + I * 2 + 4 + 2 * I * 2 + 4)
    if w["whole_pass"]:
        rw, rt, res = w["rw"], w["rt"], w["res"]
        rxb, rpb, rgb = bits(rw["x"]), bits(rw["probs"]), bits(rw["grad_out"])
        e = oracle.router_weight_fwd(rxb, oracle.BF16, rpb, oracle.BF16)
        pm, pr = bits(rt.permutation_map), bits(rt.probs)
        init = np.zeros((rt.max_rows, W), np.uint16)
        for act, x in ((oracle.SQRELU, w["ax"]), (oracle.SQRELU_CLAMP, w["ax"]),
                       (oracle.SWIGLU, w["ax2"])):
            oracle.act_with_probs_permuted(act, bits(x), init, pm, rt.n_used, pr, W,
                                           PERMUTED["scale"], True)
        oracle.unpermute_ordered(bits(w["eo"]), oracle.BF16, bits(rt.inverse_map), rt.tokens,
                                 np.zeros((rt.tokens, Hu), np.uint16), oracle.BF16)
        ee = bits(res["expert_output"]).copy()
        ee[: min(ee.shape[0], e.shape[0])] = e[: ee.shape[0]]
        oracle.residual_add(ee, bits(res["shared_expert_output"]), bits(res["residual"]),
                            oracle.BF16)
        oracle.router_weight_bwd(rgb, oracle.BF16, rxb, oracle.BF16, rpb)
        live = rt.tokens * rt.top_k
        Rr, Rs, T = w["Rr"], w["Rs"], w["T"]
        meta = 4 * rt.n_used + 4 * live
        nbytes += (Rr * ROUTER["hidden"] * 4 + Rr * 4 + Rr * ROUTER["hidden"] * 6 + Rr * 8
                   + 2 * (live * W * 2 + rt.n_used * W * 2 + meta)
                   + (live * 2 * W * 2 + rt.n_used * W * 2 + meta)
                   + live * Hu * 2 + T * rt.experts * 4 + T * Hu * 2
                   + 4 * Rs * RESIDUAL["hidden"] * 2)
    oracle.swiglu_clamped_bwd(xb, pb, gb, L)
    return nbytes


def _time_oracle(frac, steps, whole_pass=False):
    w = cpu_sample_workload(frac, whole_pass=whole_pass)
    t0 = time.perf_counter()
    b = 0
    for _ in range(steps):
        b += oracle_step(w)
    return b, time.perf_counter() - t0, w


def cpu_baseline(frac, steps=1, all_cores=True):
    """The oracle on the host, on the headline's workload: single-threaded on
    the first `frac` of the SwiGLU rows, `steps` passes, and (all_cores) the
    same fraction split over one process per host core; `step` is the whole
    pass on one core (the first quarter, at most, of every op's rows)."""
    b, dt, w = _time_oracle(frac, steps)
    out = {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "seconds": round(dt, 2), "host_cpu": _cpu_model(), "host_nproc": os.cpu_count(),
           "sample": f"clamped SwiGLU fwd+bwd on the first {w['R']} of the {SWIGLU['rows']} "
                     f"rows (inter {SWIGLU['inter']}, L {SWIGLU['limit']:g}), {steps} pass(es); "
                     "single-threaded C oracle, -O2"}
    del w
    if all_cores and (os.cpu_count() or 1) > 1:
        out["all_cores"] = oracle_pool(frac, os.cpu_count(), warmup=1, steps=max(1, steps))
    fs = min(frac, 0.25)
    b, dt, w = _time_oracle(fs, 1, whole_pass=True)
    out["step"] = {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": 1,
                   "seconds": round(dt, 2),
                   "sample": f"first {fs:g} of the rows/tokens of every op of the step "
                             f"(swiglu rows {w['R']}, router rows {w['Rr']}, tokens {w['T']}, "
                             f"residual rows {w['Rs']}); single-threaded C oracle"}
    return out


def _oracle_worker(frac, seed, warmup, steps, barrier_, q):
    """One process of the host pool: its own sample, warm-up passes, then the
    timed passes started together with the other processes."""
    try:
        w = cpu_sample_workload(frac, seed)
        for _ in range(warmup):
            oracle_step(w)
        barrier_.wait(timeout=600)
        t0 = time.perf_counter()
        b = 0
        for _ in range(steps):
            b += oracle_step(w)
        q.put((b, time.perf_counter() - t0, None))
    except Exception as e:  # reported to the parent, which raises
        q.put((0, 0.0, repr(e)))


def oracle_pool(frac_total, n, warmup=1, steps=1):
    """The oracle as it stands on `n` host processes (spawned), each on its own
    seeded sample of frac_total / n of the SwiGLU rows: aggregate GB/s = all
    processes' algorithmic bytes / the slowest process's time."""
    import multiprocessing as mp
    import oracle
    oracle.build()                       # built once here, loaded by every process
    ctx = mp.get_context("spawn")
    barrier_ = ctx.Barrier(n + 1)
    q = ctx.Queue()
    procs = [ctx.Process(target=_oracle_worker,
                         args=(frac_total / n, 7919 * (i + 1), warmup, steps, barrier_, q))
             for i in range(n)]
    for p in procs:
        p.start()
    try:
        barrier_.wait(timeout=600)
        res = [q.get(timeout=1200) for _ in range(n)]
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    errs = [e for _, _, e in res if e]
    if errs:
        raise RuntimeError(f"oracle pool: {errs[0]}")
    b = sum(r[0] for r in res)
    dt = max(r[1] for r in res)
    return {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": n, "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"{n} processes, each its own seeded sample of {frac_total / n:.4g} of the "
                      f"SwiGLU rows ({frac_total:g} in total), {steps} timed pass(es) of fwd+bwd "
                      "after a warm-up; single-threaded C oracle in each"}


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def reference_fraction(args, cores=1) -> float:
    """Fraction of the SwiGLU rows the oracle runs per step in the reference
    arm (split over `cores` processes): --cpu-sample if given, else sized so
    that the warm-up and timed steps take about two minutes on a host that
    needs ~4 s of one core per full fwd + bwd, capped at half the rows."""
    if args.cpu_sample is not None:
        return args.cpu_sample
    return max(0.005, min(0.5, 120.0 * cores / (4.0 * max(1, args.steps + args.warmup))))


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on every host core (one
    process per core, each on its share of the sampled rows)."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    n = max(1, os.cpu_count() or 1)
    args.cpu_sample = reference_fraction(args, n)
    pool = oracle_pool(args.cpu_sample, n, warmup=args.warmup, steps=args.steps)
    value = pool["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(pool["seconds"] / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": HEADLINE_NAME, "sample_fraction": args.cpu_sample},
        "cpu_baseline": pool,
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20,
                    help="pipelined end-to-end steps (fill and drain of the copy pipeline "
                         "are amortised over them)")
    ap.add_argument("--cpu-sample", type=float, default=None,
                    help="fraction of the SwiGLU rows the CPU oracle runs (default: all of "
                         "them, 3 passes, for the cpu_baseline; sized to the step count for "
                         "the reference arm)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--event-every", type=int, default=10,
                    help="per-kernel CUDA events on every N-th timed step (event records "
                         "between kernels stop programmatic launch overlap)")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the separately timed ops beyond the step")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the separately timed configurations beyond the step")
    ap.add_argument("--no-collectives", action="store_true",
                    help="with N > 1: skip the cross-rank reduce-scatter and EP combine")
    ap.add_argument("--kernel", default=None,
                    help="comma-separated kernels to run alone (profiling); default: the whole step")
    ap.add_argument("--scale", type=float, default=1.0,
                    help="row-count scale of the workload (profiling captures); default 1")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        raise SystemExit("--warmup must be >= 3")
    _, _, world = dist_env()
    if world != args.gpus and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
