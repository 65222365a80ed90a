"""Seeded synthetic inputs for the MoE expert-epilogue ops.

This module only draws inputs: it holds none of the ops' arithmetic.  The same
tensors feed the CUDA path and the CPU oracle (as raw bits).  Every generator
takes a seed and a device and uses a ``torch.Generator`` on that device, so a
(seed, device) pair always yields the same tensors.

The shapes and value distributions are those of the pages' workloads:

* clamped SwiGLU (nemo_automodel.components.moe.swiglu_triton): x = [gate | up]
  bf16 [rows, 2*inter], fp32 probs [rows, 1], bf16 grad_y [rows, inter];
* router-weight multiply (nemo_automodel.components.moe.optimized_ops):
  expert outputs [tokens, hidden], probs [tokens, 1];
* batch-invariant permuted activation and unpermute
  (core.inference.moe.batch_invariant): top-k routing over E experts, rows
  grouped by expert and padded to the grouped-GEMM alignment;
* residual add (core.fusions.fused_moe_residual_add): three same-shape tensors;
* rank-order reduce-scatter (core.inference.moe.batch_invariant,
  ordered_reduce_scatter_v): every EP rank's partial outputs for the tokens of
  all ranks, each rank owning a ragged, contiguous block of token rows;
* EP combine (the same page's unpermute followed by the reduce-scatter): the
  top-k routing of the tokens of all ranks over world x experts-per-rank
  experts, each rank holding its own experts' expert-grouped rows.
"""
from __future__ import annotations

import dataclasses

import torch

NAN_BF16 = 0x7FC0  # quiet NaN bits used as "never read" sentinels


def _gen(seed: int, device) -> torch.Generator:
    return torch.Generator(device=device).manual_seed(int(seed))


def normal(shape, sigma, gen, device, dtype=torch.bfloat16):
    """N(0, sigma^2) drawn in fp32 and stored in ``dtype``."""
    return (torch.randn(*shape, generator=gen, device=device) * sigma).to(dtype)


def uniform(shape, lo, hi, gen, device):
    return torch.rand(*shape, generator=gen, device=device) * (hi - lo) + lo


def topk_softmax_weights(tokens, experts, top_k, gen, device):
    """Router weights: softmax over the top-k of N(0,1) logits per token.
    Returns (weights fp32 [tokens, top_k], expert ids int64 [tokens, top_k])."""
    logits = torch.randn(tokens, experts, generator=gen, device=device)
    top_v, top_i = logits.topk(top_k, dim=-1)
    return torch.softmax(top_v, dim=-1), top_i


# ------------------------------------------------------------------ SwiGLU

def swiglu_inputs(rows, inter, *, sigma=2.0, probs="uniform", top_k=8, experts=64,
                  limit=None, plant_ties=False, seed=0, device="cpu"):
    """x bf16 [rows, 2*inter] ~ N(0, sigma^2); probs fp32 [rows, 1] either
    U(0, 1) or top-k softmax weights flattened token-major; grad_y bf16
    [rows, inter] ~ N(0, 1).

    With ``plant_ties`` and a finite ``limit`` some entries are set exactly to
    the clamp bounds (gate == L, up == -L, up == +L) and some just above
    (the next bf16 after L), so both sides of each inclusive mask occur."""
    g = _gen(seed, device)
    x = normal((rows, 2 * inter), sigma, g, device)
    if probs == "uniform":
        p = uniform((rows, 1), 0.0, 1.0, g, device)
    elif probs == "topk_softmax":
        if rows % top_k:
            raise ValueError("rows must be a multiple of top_k")
        w, _ = topk_softmax_weights(rows // top_k, experts, top_k, g, device)
        p = w.reshape(rows, 1).contiguous()
    else:
        raise ValueError(probs)
    grad_y = normal((rows, inter), 1.0, g, device)
    if plant_ties and limit is not None and limit != float("inf"):
        L = torch.tensor(limit, dtype=torch.bfloat16)
        if float(L) != float(limit):
            raise ValueError("plant_ties needs a limit that bf16 represents exactly")
        above = (L.view(torch.int16) + 1).view(torch.bfloat16)  # next bf16 after L
        sel = torch.randint(0, 6, (rows, inter), generator=g, device=device)
        gate, up = x[:, :inter], x[:, inter:]
        gate[sel == 0] = L.to(device)
        gate[sel == 1] = above.to(device)
        up[sel == 2] = L.to(device)
        up[sel == 3] = (-L).to(device)
        up[sel == 4] = (-above).to(device)
    return {"x": x, "probs": p, "grad_y": grad_y}


# ------------------------------------------------------- router weight

def router_weight_inputs(rows, hidden, *, out_dtype=torch.bfloat16, seed=0, device="cpu"):
    """x bf16 [rows, hidden] ~ N(0,1); probs fp32 [rows, 1] ~ U(0.01, 1);
    grad_out ~ N(0,1) drawn as bf16 and stored in out_dtype (so the bf16 and
    fp32 output runs share values)."""
    g = _gen(seed, device)
    x = normal((rows, hidden), 1.0, g, device)
    p = uniform((rows, 1), 0.01, 1.0, g, device)
    grad_out = normal((rows, hidden), 1.0, g, device).to(out_dtype)
    return {"x": x, "probs": p, "grad_out": grad_out}


# ------------------------------------------------------- routing / permutation

@dataclasses.dataclass
class Routing:
    """Expert-grouped, alignment-padded layout of top-k routed tokens.

    permutation_map int32 [max_rows]: for a live row, the flat token-major
      index t*top_k + k of its routing weight; -1 for a padding row (and for
      every row at or past n_used).
    inverse_map int32 [tokens, experts]: the row holding (t, e), or -1.
    probs fp32 [tokens*top_k]: routing weights, token-major.
    n_used: rows in the padded live prefix (sum over experts of the count
      rounded up to ``align``)."""
    tokens: int
    top_k: int
    experts: int
    align: int
    max_rows: int
    n_used: int
    permutation_map: torch.Tensor
    inverse_map: torch.Tensor
    probs: torch.Tensor
    counts: torch.Tensor


def routing(tokens, top_k, experts, align, *, seed=0, device="cpu"):
    """Uniform random top-k routing (distinct experts per token, from N(0,1)
    logits), rows ordered stably by (expert, token, k), each expert's block
    padded to a multiple of ``align`` rows."""
    g = _gen(seed, device)
    w, ids = topk_softmax_weights(tokens, experts, top_k, g, device)
    flat_expert = ids.reshape(-1)
    order = torch.sort(flat_expert, stable=True).indices          # flat ids by expert
    counts = torch.bincount(flat_expert, minlength=experts)
    padded = (counts + align - 1) // align * align
    pad_start = torch.cumsum(padded, 0) - padded
    cnt_start = torch.cumsum(counts, 0) - counts
    sorted_expert = flat_expert[order]
    rows_of_sorted = pad_start[sorted_expert] + (
        torch.arange(order.numel(), device=device) - cnt_start[sorted_expert])
    max_rows = tokens * top_k + experts * align
    pmap = torch.full((max_rows,), -1, dtype=torch.int32, device=device)
    pmap[rows_of_sorted] = order.to(torch.int32)
    inv = torch.full((tokens, experts), -1, dtype=torch.int32, device=device)
    tok = order // top_k
    inv[tok, sorted_expert] = rows_of_sorted.to(torch.int32)
    return Routing(tokens, top_k, experts, align, max_rows, int(padded.sum()), pmap, inv,
                   w.reshape(-1).contiguous(), counts)


def permuted_activation_input(rt: Routing, width, *, swiglu, sigma=2.0, seed=1,
                              device="cpu"):
    """Grouped-GEMM FC1 output [max_rows, width] (or [max_rows, 2*width] for
    SwiGLU) ~ N(0, sigma^2).  Padding rows and rows past n_used hold NaN
    sentinels: the op must never read them."""
    g = _gen(seed, device)
    cols = 2 * width if swiglu else width
    x = normal((rt.max_rows, cols), sigma, g, device)
    dead = rt.permutation_map < 0
    x.view(torch.int16)[dead] = NAN_BF16
    return x


def expert_output_input(rt: Routing, hidden, *, dtype=torch.bfloat16, seed=2, device="cpu"):
    """Grouped-GEMM FC2 output [max_rows, hidden] ~ N(0,1); padding rows and
    rows past n_used are NaN sentinels."""
    g = _gen(seed, device)
    eo = normal((rt.max_rows, hidden), 1.0, g, device, dtype=dtype)
    eo[rt.permutation_map < 0] = float("nan")
    return eo


# ------------------------------------------------------------ residual add

def residual_inputs(shape, dtype, *, seed=0, device="cpu"):
    """expert_output, shared_expert_output, residual ~ N(0,1) in ``dtype``."""
    g = _gen(seed, device)
    return {k: normal(shape, 1.0, g, device, dtype=dtype)
            for k in ("expert_output", "shared_expert_output", "residual")}


# --------------------------------------------------- raw-bit views (numpy)

@dataclasses.dataclass
class ReduceScatterCase:
    """world buffers [capacity_rows, hidden] (rank order); rank q's tokens are
    rows [rank_token_offset[q], rank_token_offset[q] + counts[q]); ep_tokens =
    sum(counts) rows hold data, the rest of each buffer is NaN ("never read")."""
    buffers: list
    rank_token_offset: torch.Tensor   # int32 [world]
    counts: list
    ep_tokens: int


def reduce_scatter_inputs(world, tokens, hidden, *, dtype=torch.bfloat16, spare_rows=0,
                          sigma=1.0, seed=0, device="cpu") -> ReduceScatterCase:
    """`tokens` token rows split over `world` ranks by a uniform multinomial
    draw (ragged counts, some possibly zero); partials ~ N(0, sigma^2) drawn in
    fp32 and stored in `dtype`; `spare_rows` NaN rows past the data."""
    g = _gen(seed, device)
    owner = torch.randint(0, world, (tokens,), generator=g, device=device)
    counts = torch.bincount(owner, minlength=world).tolist()
    offsets = [0]
    for c in counts[:-1]:
        offsets.append(offsets[-1] + c)
    cap = tokens + spare_rows
    bufs = []
    for _ in range(world):
        b = torch.full((cap, hidden), float("nan"), dtype=dtype, device=device)
        b[:tokens] = (torch.randn(tokens, hidden, generator=g, device=device) * sigma).to(dtype)
        bufs.append(b)
    return ReduceScatterCase(bufs, torch.tensor(offsets, dtype=torch.int32, device=device),
                             counts, tokens)


@dataclasses.dataclass
class EpCombineCase:
    """Per rank q (rank order): expert_outputs[q] [max_rows, hidden], the rows of
    its experts (expert-grouped, padded; NaN past its rows), and inverse_maps[q]
    int32 [tokens, experts_per_rank] over the tokens of all ranks (row in
    expert_outputs[q], or -1).  Rank q owns tokens [rank_token_offset[q],
    + counts[q])."""
    expert_outputs: list
    inverse_maps: list
    rank_token_offset: torch.Tensor
    counts: list
    tokens: int
    max_rows: int
    routing: Routing


def ep_combine_inputs(world, tokens, top_k, experts_per_rank, align, hidden, *,
                      dtype=torch.bfloat16, seed=0, device="cpu") -> EpCombineCase:
    """Expert parallelism over `world` ranks: uniform top-k routing over
    world * experts_per_rank experts (distinct per token); rank q hosts experts
    [q * experts_per_rank, (q + 1) * experts_per_rank); expert outputs ~ N(0,1);
    tokens split over the ranks by a uniform multinomial draw."""
    E = world * experts_per_rank
    rt = routing(tokens, top_k, E, align, seed=seed, device=device)
    eo = expert_output_input(rt, hidden, dtype=dtype, seed=seed + 1, device=device)
    padded = (rt.counts + align - 1) // align * align
    starts = torch.cumsum(padded, 0) - padded
    bounds = []
    for q in range(world):
        e0, e1 = q * experts_per_rank, (q + 1) * experts_per_rank
        bounds.append((int(starts[e0]), int(starts[e1 - 1] + padded[e1 - 1])))
    max_rows = max(1, max(r1 - r0 for r0, r1 in bounds))
    eos, invs = [], []
    for q, (r0, r1) in enumerate(bounds):
        blk = torch.full((max_rows, hidden), float("nan"), dtype=dtype, device=device)
        blk[:r1 - r0] = eo[r0:r1]
        eos.append(blk)
        inv = rt.inverse_map[:, q * experts_per_rank:(q + 1) * experts_per_rank]
        invs.append(torch.where(inv >= 0, inv - r0, torch.full_like(inv, -1)).contiguous())
    g = _gen(seed + 2, device)
    owner = torch.randint(0, world, (tokens,), generator=g, device=device)
    counts = torch.bincount(owner, minlength=world).tolist()
    offsets = [0]
    for c in counts[:-1]:
        offsets.append(offsets[-1] + c)
    return EpCombineCase(eos, invs, torch.tensor(offsets, dtype=torch.int32, device=device),
                         counts, tokens, max_rows, rt)


def bits(t: torch.Tensor):
    """numpy view of a CPU tensor: uint16 bits for 16-bit floats, else as is."""
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()


def from_bits(a, dtype) -> torch.Tensor:
    """Inverse of :func:`bits`."""
    import numpy as np
    a = np.ascontiguousarray(a)
    if dtype in (torch.bfloat16, torch.float16):
        return torch.from_numpy(a.view(np.int16).copy()).view(dtype)
    return torch.from_numpy(a.copy()).to(dtype)
