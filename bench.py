#!/usr/bin/env python
"""Throughput of the MoE expert-epilogue pass on B200: achieved HBM GB/s.

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

value = algorithmic bytes of all steps on all ranks / max-over-ranks device
time (CUDA events on the launching stream, barrier + synchronize on both
sides).  Per-kernel durations come from CUDA events around each launch on
every 10th timed step (event records between kernels would stop the
programmatic launch overlap on every step).  Every kernel's working set
exceeds the 126 MB L2, so no flush is needed between steps.  Multi-GPU runs
(torchrun) are weak scaling: each rank runs the full step on its own inputs;
the only collectives are the barrier and the max of the timings.

The line also carries `e2e` (the same step through the public API with every
input copied from pinned host memory and every output copied back inside the
timed region, pipelined), `next_rows` (the bounded SwiGLU, the fused chain and
the rank-order reduce-scatter, timed after the step), `clocks`, `roofline` and
`cpu_baseline` (the CPU oracle, one core and all cores).  `--impl reference`
times the CPU oracle alone on every host core.
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
ORDER = ["swiglu_fwd", "router_weight_fwd", "act_sqrelu", "act_sqrelu_clamp", "act_swiglu",
         "unpermute", "residual_add", "router_weight_bwd", "swiglu_bwd"]


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
             "unpermute_reduce_scatter")
RS_WORLD = 8  # EP ranks of the rank-order reduce-scatter, all blocks on this GPU


def measure_next_rows(device, seed, reps, peak, scale=1.0, only=None):
    """The ops beyond the step: the device-bounded weighted SwiGLU, the fused
    router-weight -> unpermute -> residual chain (against the same chain as
    three launches) and the rank-order reduce-scatter.  Timed after the step,
    outside its timed region."""
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
        out.update(_measure_ep_combine(device, seed, reps, peak, T, K, E, A, H))
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


def _measure_ep_combine(device, seed, reps, peak, T, K, E, A, H, world=RS_WORLD):
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
    return {"unpermute_reduce_scatter": {
        "shape": f"{world} ranks x {E // world} experts, {T} tokens top-{K}, hidden {H}, bf16, "
                 f"all ranks' expert rows on one GPU, one launch per rank",
        "us": round(ms_f * 1e3, 2), "bytes": nb_f, "gbs": round(nb_f / ms_f / 1e6, 1),
        "frac": round(nb_f / ms_f / 1e6 / peak, 4),
        "two_step_us": round(ms_2 * 1e3, 2), "two_step_bytes": nb_2,
        "speedup_vs_two_step": round(ms_2 / ms_f, 3)}}


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
    if only and len(only) == 1 and next(iter(only)) in NEXT_ROWS:
        # a next-row op alone (profiling captures): warm-ups, then --steps launches
        peak, _ = hbm_peak()
        res = measure_next_rows(device, 1000 * rank, args.steps, peak, args.scale,
                                only=next(iter(only)))
        if rank == 0:
            print(json.dumps({"kernel": args.kernel, "scale": args.scale, "result": res}),
                  flush=True)
        return
    if only and not only <= set(ORDER):
        raise SystemExit(f"unknown --kernel {args.kernel}; choose from {ORDER + list(NEXT_ROWS)}")
    batch = Batch(device, seed=1000 * rank, scale=args.scale, kernels=only)
    kernels = batch.kernels()
    nbytes = algorithmic_bytes(batch.rt.n_used, args.scale)
    nbytes = {n: nbytes[n] for n, _ in kernels}
    rows = rows_per_launch(args.scale)
    bytes_per_step = sum(nbytes.values())
    stream = torch.cuda.current_stream(device)

    for _ in range(args.warmup):
        for _, fn in kernels:
            fn()
    torch.cuda.synchronize(device)

    K = args.steps
    every = max(1, args.event_every)
    probed = [k for k in range(K) if k % every == every - 1] or [K - 1]
    ev = {name: {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for k in probed} for name, _ in kernels}
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(device.index) if not args.no_clocks else contextlib.nullcontext()
    with sampler:
        barrier(device)
        torch.cuda.synchronize(device)
        t_start.record(stream)
        for k in range(K):
            if k in probed:                # per-kernel events on every `every`-th step
                for name, fn in kernels:
                    ev[name][k][0].record(stream)
                    fn()
                    ev[name][k][1].record(stream)
            else:
                for _, fn in kernels:
                    fn()
        t_end.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
    elapsed_ms = t_start.elapsed_time(t_end)
    max_ms = max_over_ranks(elapsed_ms, device)
    clocks = sampler.summary() if not args.no_clocks else None

    per_kernel = {}
    peak, peak_kind = hbm_peak()
    for name, _ in kernels:
        times = sorted(a.elapsed_time(b) for a, b in ev[name].values())
        avg_ms = sum(times) / len(times)
        gbs = nbytes[name] / (avg_ms * 1e-3) / 1e9
        per_kernel[name] = {"us": round(avg_ms * 1e3, 2), "median_us": round(times[len(times) // 2] * 1e3, 2),
                            "bytes": nbytes[name], "gbs": round(gbs, 1),
                            "frac": round(gbs / peak, 4),
                            "share": None}
        if rows[name]:
            per_kernel[name]["rows_per_s"] = rows[name] / (avg_ms * 1e-3)
    total_kernel_ms = sum(v["us"] for v in per_kernel.values())
    for v in per_kernel.values():
        v["share"] = round(v["us"] / total_kernel_ms, 4)
    dominant = max(per_kernel, key=lambda n: per_kernel[n]["us"])
    d = per_kernel[dominant]

    e2e = None
    if not args.no_e2e and not args.kernel:
        e2e = run_e2e(batch, nbytes, args, device, 1000 * rank)
    n_used, n_kernels = batch.rt.n_used, len(kernels)
    next_rows = None
    if not args.kernel and not args.no_next_rows:
        del batch, kernels
        torch.cuda.empty_cache()
        next_rows = measure_next_rows(device, 1000 * rank, 20, peak)

    sw = None
    if "swiglu_fwd" in per_kernel and "swiglu_bwd" in per_kernel:
        sw_bytes = nbytes["swiglu_fwd"] + nbytes["swiglu_bwd"]
        sw_us = per_kernel["swiglu_fwd"]["us"] + per_kernel["swiglu_bwd"]["us"]
        sw_gbs = sw_bytes / (sw_us * 1e-6) / 1e9
        sw = {"gbs": round(sw_gbs, 1), "frac": round(sw_gbs / peak, 4),
              "rows_per_s": rows["swiglu_fwd"] / (sw_us * 1e-6),
              "fwd_frac": per_kernel["swiglu_fwd"]["frac"],
              "bwd_frac": per_kernel["swiglu_bwd"]["frac"]}
    workload = WORKLOAD_NAME if not args.kernel and args.scale == 1.0 else \
        f"{args.kernel or 'all'} at scale {args.scale:g} of: {WORKLOAD_NAME}"
    line = {
        "metric": METRIC,
        "value": round(aggregate_value(bytes_per_step, K, world, max_ms * 1e-3), 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(max_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload, "bytes_per_step": bytes_per_step,
                   "l2": "no flush: every kernel streams > 126 MB (inputs larger than L2)",
                   "parallelism": f"weak: {world} independent replica(s), one per GPU",
                   "per_kernel_events": f"on {len(probed)} of the {K} timed steps (every "
                                        f"{every}th); the other steps run without event records",
                   "n_used": n_used},
        "swiglu_fwd_bwd": sw,
        "roofline": {"kernel": dominant, "bound": "hbm", "achieved": d["gbs"], "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": d["frac"],
                     "algorithmic_bytes": d["bytes"],
                     "traffic": ncu_traffic(dominant) if args.scale == 1.0 else None},
        "kernels": per_kernel,
        "gpu_launches": K * n_kernels,
        "clocks": clocks,
        "e2e": e2e,
        "next_rows": next_rows,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.kernel:
        line["cpu_baseline"] = cpu_baseline(args.cpu_sample or 0.25, steps=1)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(batch, nbytes, args, device, seed):
    """The same step through the public API with inputs in pinned host memory:
    every step copies all of its inputs host -> device, runs the kernels and
    copies all of its outputs device -> host, all inside the timed region.
    Steps are pipelined as a user would drive them: two device buffer sets,
    a copy-in stream, the compute stream and a copy-out stream, so step k's
    kernels overlap step k+1's inputs and step k-1's outputs on the host link.
    Events order every reuse of a buffer set."""
    sets = [batch, Batch(device, seed=seed + 7, scale=args.scale)]
    kernel_sets = [b.kernels() for b in sets]
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
    return {"value": round(aggregate_value(sum(nbytes.values()), n, world, ms * 1e-3), 2),
            "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "ms_per_step": round(ms / n, 3),
            "pipeline": "2 device buffer sets; copy-in, compute and copy-out streams"}


# ---------------------------------------------------------------- CPU oracle

def cpu_sample_workload(frac: float, seed: int = 0):
    """A bounded sample of the same workload on the host: the first `frac` of
    the rows (tokens) of every op, same distributions."""
    import numpy as np  # noqa: F401
    from moe_expert_epilogue_b200 import inputs
    R = max(8, int(SWIGLU["rows"] * frac) // 8 * 8)
    Rr = max(1, int(ROUTER["rows"] * frac))
    T = max(8, int(PERMUTED["tokens"] * frac))
    Rs = max(1, int(RESIDUAL["rows"] * frac))
    sw = inputs.swiglu_inputs(R, SWIGLU["inter"], sigma=SWIGLU["sigma"], probs="topk_softmax",
                              seed=seed)
    rw = inputs.router_weight_inputs(Rr, ROUTER["hidden"], seed=seed + 1)
    rt = inputs.routing(T, PERMUTED["top_k"], PERMUTED["experts"], PERMUTED["align"], seed=seed + 2)
    ax = inputs.permuted_activation_input(rt, PERMUTED["width"], swiglu=False, seed=seed + 3)
    ax2 = inputs.permuted_activation_input(rt, PERMUTED["width"], swiglu=True, seed=seed + 4)
    eo = inputs.expert_output_input(rt, PERMUTED["hidden"], seed=seed + 5)
    res = inputs.residual_inputs((Rs, RESIDUAL["hidden"]), torch.bfloat16, seed=seed + 6)
    return dict(R=R, Rr=Rr, T=T, Rs=Rs, sw=sw, rw=rw, rt=rt, ax=ax, ax2=ax2, eo=eo, res=res)


def oracle_step(w):
    """One pass of the oracle over the sampled workload; returns its algorithmic bytes."""
    import numpy as np
    import oracle
    from moe_expert_epilogue_b200.inputs import bits
    L, I, W, Hu = SWIGLU["limit"], SWIGLU["inter"], PERMUTED["width"], PERMUTED["hidden"]
    sw, rw, rt, res = w["sw"], w["rw"], w["rt"], w["res"]
    xb, pb, gb = bits(sw["x"]), bits(sw["probs"]), bits(sw["grad_y"])
    oracle.swiglu_clamped_fwd(xb, pb, L)
    rxb, rpb, rgb = bits(rw["x"]), bits(rw["probs"]), bits(rw["grad_out"])
    e = oracle.router_weight_fwd(rxb, oracle.BF16, rpb, oracle.BF16)
    pm, pr = bits(rt.permutation_map), bits(rt.probs)
    init = np.zeros((rt.max_rows, W), np.uint16)
    for act, x in ((oracle.SQRELU, w["ax"]), (oracle.SQRELU_CLAMP, w["ax"]), (oracle.SWIGLU, w["ax2"])):
        oracle.act_with_probs_permuted(act, bits(x), init, pm, rt.n_used, pr, W, PERMUTED["scale"],
                                       True)
    oracle.unpermute_ordered(bits(w["eo"]), oracle.BF16, bits(rt.inverse_map), rt.tokens,
                             np.zeros((rt.tokens, Hu), np.uint16), oracle.BF16)
    ee = bits(res["expert_output"]).copy()
    ee[: min(ee.shape[0], e.shape[0])] = e[: ee.shape[0]]
    oracle.residual_add(ee, bits(res["shared_expert_output"]), bits(res["residual"]), oracle.BF16)
    oracle.router_weight_bwd(rgb, oracle.BF16, rxb, oracle.BF16, rpb)
    oracle.swiglu_clamped_bwd(xb, pb, gb, L)
    live = rt.tokens * rt.top_k
    R, Rr, Rs, T = w["R"], w["Rr"], w["Rs"], w["T"]
    meta = 4 * rt.n_used + 4 * live
    return (R * (2 * I * 2 + 4 + I * 2) + R * (2 * I * 2 + I * 2 + 4 + 2 * I * 2 + 4)
            + Rr * ROUTER["hidden"] * 4 + Rr * 4 + Rr * ROUTER["hidden"] * 6 + Rr * 8
            + 2 * (live * W * 2 + rt.n_used * W * 2 + meta)
            + (live * 2 * W * 2 + rt.n_used * W * 2 + meta)
            + live * Hu * 2 + T * rt.experts * 4 + T * Hu * 2
            + 4 * Rs * RESIDUAL["hidden"] * 2)


def cpu_baseline(frac, steps=1, all_cores=True):
    """The oracle on the host: single-threaded on the first `frac` of every
    op's rows, and (all_cores) the same fraction split over one process per
    host core."""
    w = cpu_sample_workload(frac)
    t0 = time.perf_counter()
    b = 0
    for _ in range(steps):
        b += oracle_step(w)
    dt = time.perf_counter() - t0
    out = {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "seconds": round(dt, 2), "host_cpu": _cpu_model(), "host_nproc": os.cpu_count(),
           "sample": f"first {frac:g} of the rows/tokens of every op of the step "
                     f"(swiglu rows {w['R']}, router rows {w['Rr']}, tokens {w['T']}, "
                     f"residual rows {w['Rs']}); single-threaded C oracle, -O2"}
    del w
    if all_cores and (os.cpu_count() or 1) > 1:
        out["all_cores"] = oracle_pool(frac, os.cpu_count(), warmup=1, steps=4 * max(1, steps))
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
    seeded sample of frac_total / n of every op's rows: aggregate GB/s = all
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
                      f"rows/tokens of every op ({frac_total:g} in total), {steps} timed "
                      "pass(es) after a warm-up; single-threaded C oracle in each"}


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def reference_fraction(args, cores=1) -> float:
    """Row fraction of every op the oracle runs per step in the reference arm
    (split over `cores` processes): --cpu-sample if given, else sized so that
    the warm-up and timed steps take about two minutes on a host that needs
    ~17 s of one core per full step, capped at half the workload (host memory)."""
    if args.cpu_sample is not None:
        return args.cpu_sample
    return max(0.005, min(0.5, 120.0 * cores / (17.0 * max(1, args.steps + args.warmup))))


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
        "config": {"workload": WORKLOAD_NAME, "sample_fraction": args.cpu_sample},
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
                    help="fraction of the rows of every op the CPU oracle runs (default: "
                         "0.25 for the cpu_baseline; sized to the step count for the "
                         "reference arm)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--event-every", type=int, default=10,
                    help="per-kernel CUDA events on every N-th timed step (event records "
                         "between kernels stop programmatic launch overlap)")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the separately timed ops beyond the step")
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
