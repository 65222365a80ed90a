/*
 * moe_epilogue.h -- C ABI of the B200 (sm_100a) MoE expert-epilogue library.
 *
 * The memory-bound ops that sit between the grouped GEMMs of a
 * Mixture-of-Experts layer and the residual stream (the seven of the hot path,
 * their dtype variants, the bounded SwiGLU, the fused epilogue chain and the
 * rank-order reduce-scatter), plus the IPC helpers under the reduce-scatter.
 * Each op entry point takes caller-owned DEVICE pointers, sizes and a CUDA
 * stream, validates its arguments on the host, enqueues exactly one kernel on
 * `stream` and returns.
 *
 * Common contract
 *   - Ownership: every pointer is owned by the caller and must stay valid
 *     until the enqueued kernel has finished.  The op entry points allocate
 *     nothing, keep no per-call state and never synchronise, so calls may be
 *     captured in a CUDA graph.  (Only moe_symm_alloc and moe_ipc_open create
 *     anything; the caller releases it with moe_symm_free / moe_ipc_close.)
 *   - Layout: 2-D tensors are row-major.  `ld_*` arguments are leading
 *     dimensions in ELEMENTS (the distance between the starts of two rows);
 *     where no leading dimension is taken, rows are contiguous.
 *   - Counts that change at run time (n_used, valid_tokens, bound_elems,
 *     ep_tokens, rank offsets) live in DEVICE memory, read by the kernel, so
 *     a captured graph stays valid as they change.  The matching maximum sizes
 *     are host arguments.
 *   - Alignment: every pointer must be aligned to its element size
 *     (MOE_ERR_ALIGN otherwise).  16-byte aligned pointers and leading
 *     dimensions / widths that are multiples of 8 elements take the
 *     vectorised path (for 16-bit data, 32-byte aligned pointers and widths
 *     that are multiples of 16 take 32-byte accesses where that is faster);
 *     anything else takes an element-wise path inside the same kernel family
 *     with identical results (grad_probs, a reduction: within its stated
 *     tolerance, its order fixed for a given layout).
 *   - Aliasing: outputs must not overlap inputs, except that
 *     moe_residual_add and moe_epilogue_fused may run in place
 *     (out == residual).
 *   - Errors: the return value is MOE_OK or one of the MOE_ERR_* codes below.
 *     Argument errors are detected before anything is enqueued.  MOE_ERR_CUDA
 *     means a CUDA runtime call failed (moe_last_cuda_error() gives the
 *     cudaError_t); note that an asynchronous error left pending by earlier
 *     work on the device can surface here too.  Sizes of zero are valid
 *     no-ops, except that a probability gradient over zero columns is still
 *     written: the empty sum, +0.
 *   - Device error word: the ops that read counts or routing metadata from
 *     device memory take an optional `int32_t* dev_err` (device memory, may
 *     be NULL).  Out-of-range metadata never causes an out-of-bounds access:
 *     the kernel clamps or skips and ORs MOE_DEVERR_* bits into *dev_err.
 *   - Numerics: inputs are widened to fp32, the documented formula is
 *     evaluated in fp32 and each output is rounded once to its dtype with
 *     round-to-nearest-even (the fused chain keeps each rounding of the
 *     three steps it fuses).  Every result is independent of the grid size,
 *     of the other rows / tokens in the batch and of the run (no atomics in
 *     any reduction).
 *
 * Sources (API reference pages, cited by page title and documented symbol):
 *   [OPT] nemo_automodel.components.moe.optimized_ops
 *   [SWI] nemo_automodel.components.moe.swiglu_triton
 *   [BI]  core.inference.moe.batch_invariant
 *   [RES] core.fusions.fused_moe_residual_add
 */
#ifndef MOE_EPILOGUE_H
#define MOE_EPILOGUE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MOE_BF16 = 0, MOE_FP16 = 1, MOE_FP32 = 2 } moe_dtype;

typedef enum {
  MOE_ACT_SQRELU = 0,       /* squared ReLU, square rounded to bf16 first        */
  MOE_ACT_SQRELU_CLAMP = 1, /* tanh soft clamp, then squared ReLU, all in fp32   */
  MOE_ACT_SWIGLU = 2        /* silu(gate) * up, gate = first half of the row     */
} moe_act;

enum {
  MOE_OK = 0,
  MOE_ERR_NULL = 1,  /* a required pointer is NULL                              */
  MOE_ERR_SHAPE = 2, /* negative size, leading dim below the row width, or a
                        size beyond the documented maximum                     */
  MOE_ERR_DTYPE = 3, /* dtype (or activation) not supported for that argument   */
  MOE_ERR_ALIGN = 4, /* a pointer not aligned to its element size               */
  MOE_ERR_LIMIT = 5, /* limit or clamp_scale not a positive number              */
  MOE_ERR_CUDA = 6   /* a CUDA runtime call or the launch failed                */
};

/* Bits ORed into the optional device error word. */
enum {
  MOE_DEVERR_COUNT = 1,  /* *n_used / *valid_tokens outside [0, max]: clamped    */
  MOE_DEVERR_MAP = 2,    /* permutation_map entry >= num_probs: row skipped       */
  MOE_DEVERR_INVERSE = 4, /* inverse_map entry >= max_rows: contribution skipped  */
  MOE_DEVERR_TIMEOUT = 8  /* a kernel's barrier wait gave up (~1 s: a shared-memory
                             copy or a consumer that never completed).  The rows the
                             waiting warps had not reached were not written.  Before
                             exiting, a CTA waits (bounded again) for every copy it
                             issued; if that wait gives up as well, a copy may land in
                             shared memory after the CTA has exited, where another
                             kernel's CTA may live.  Treat the bit as fatal for the
                             results of everything enqueued after the call on the
                             device: discard them and rebuild the CUDA context.     */
};

/* Human-readable name of a status code (static storage). */
MOE_API const char* moe_status_string(int status);

/* cudaError_t of the most recent MOE_ERR_CUDA on the calling thread (0 if none). */
MOE_API int moe_last_cuda_error(void);

/* Library ABI version, currently 1. */
MOE_API int moe_abi_version(void);

/* Error bits recorded on the current device by calls that were given no
 * error word of their own (today: the TMA-staged clamped-SwiGLU forward
 * through moe_swiglu_clamped_fwd, or _ex with dev_err NULL:
 * MOE_DEVERR_TIMEOUT).  One word per device, shared by every stream and
 * thread; pass dev_err to moe_swiglu_clamped_fwd_ex to keep a call's bits
 * apart.  Synchronous: waits for the device, copies the word into *bits and,
 * if `clear`, resets it.  Returns MOE_OK, MOE_ERR_NULL or MOE_ERR_CUDA. */
MOE_API int moe_device_errors(int32_t* bits, int clear);

/* ------------------------------------------------------------------------
 * Clamped, probability-weighted SwiGLU, forward.
 * [SWI] module docstring and the forward kernel (_swiglu_clamped_fwd_kernel):
 *   y[r, j] = silu(clamp(g, max=L)) * clamp(u, -L, L) * probs[r]
 *   with g = x[r, j], u = x[r, inter + j], silu(z) = z * sigmoid(z);
 *   fp32 math, one rounding to dt.  clamp is torch.clamp (NaN propagates).
 * x      dt [rows, ld_x], columns [0, inter) gate, [inter, 2*inter) up; ld_x >= 2*inter
 * probs  fp32 [rows] (one routing probability per row, i.e. [rows, 1])
 * y      dt [rows, ld_y], ld_y >= inter; columns >= inter are not written
 * limit  L > 0, may be +inf (no clamping); NaN or <= 0 -> MOE_ERR_LIMIT
 * dt     storage dtype of x and y: MOE_BF16, MOE_FP16 or MOE_FP32 (the page's
 *        _SUPPORTED_DTYPES)
 * ---------------------------------------------------------------------- */
MOE_API int moe_swiglu_clamped_fwd(const void* x, const float* probs, void* y, int64_t rows,
                           int64_t inter, int64_t ld_x, int64_t ld_y, float limit,
                           moe_dtype dt, cudaStream_t stream);

/* moe_swiglu_clamped_fwd with an error word of the caller's: dev_err
 * (optional int32, device memory, 4-byte aligned) receives MOE_DEVERR_TIMEOUT
 * if the TMA-staged kernel (contiguous 16-byte aligned rows of at least 512
 * columns that fit its shared-memory ring: up to 6392 columns in bf16 / fp16,
 * 3192 in fp32) gave up a barrier wait; with dev_err NULL the bit
 * goes to the per-device word of moe_device_errors().  Same computation,
 * arguments and status codes as moe_swiglu_clamped_fwd. */
MOE_API int moe_swiglu_clamped_fwd_ex(const void* x, const float* probs, void* y, int64_t rows,
                                      int64_t inter, int64_t ld_x, int64_t ld_y, float limit,
                                      moe_dtype dt, int32_t* dev_err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Clamped SwiGLU, one-pass backward.
 * [SWI] module docstring and the backward kernel (_swiglu_clamped_bwd_kernel):
 *   a = dy * p,   s = silu(gc),   gc = clamp(g, max=L),  uc = clamp(u, -L, L)
 *   grad_x[r, j]         = a * uc * silu'(gc)  where g <= L,        else 0
 *   grad_x[r, inter + j] = a * s               where -L <= u <= L,  else 0
 *   grad_probs[r]        = sum_j dy * s * uc   (fp32, reduced per row)
 *   silu'(z) = sigmoid(z) * (1 + z * (1 - sigmoid(z))); the masks are
 *   torch.clamp's inclusive ranges on the input values; grad_x is rounded
 *   once to dt.  grad_probs is reduced in a fixed order (per-thread
 *   partials over a fixed column assignment, a fixed warp butterfly, warps
 *   in index order), independent of the grid and of the batch.
 * x           dt [rows, ld_x]   (the forward's input, recomputed from)
 * probs       fp32 [rows]
 * grad_y      dt [rows, ld_gy], ld_gy >= inter
 * grad_x      dt [rows, ld_gx], ld_gx >= 2*inter  (output)
 * grad_probs  fp32 [rows]                         (output; +0 when inter == 0)
 * dt          MOE_BF16, MOE_FP16 or MOE_FP32
 * ---------------------------------------------------------------------- */
MOE_API int moe_swiglu_clamped_bwd(const void* x, const float* probs, const void* grad_y,
                           void* grad_x, float* grad_probs, int64_t rows, int64_t inter,
                           int64_t ld_x, int64_t ld_gy, int64_t ld_gx, float limit,
                           moe_dtype dt, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Router-weight multiply in fp32, forward.
 * [OPT] _rw_fwd_core and _RouterWeightMulFunction.forward:
 *   out[r, h] = (x[r, h].float() * probs[r]).to(out_dtype)
 *   one fp32 multiply and one rounding: bitwise identical to the eager op.
 * x      x_dt [rows, hidden] contiguous;  x_dt in {BF16, FP16, FP32}
 * probs  fp32 [rows]
 * out    out_dt [rows, hidden] contiguous; out_dt in {BF16, FP16, FP32}
 * ---------------------------------------------------------------------- */
MOE_API int moe_router_weight_mul_fwd(const void* x, moe_dtype x_dt, const float* probs, void* out,
                              moe_dtype out_dt, int64_t rows, int64_t hidden,
                              cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Router-weight multiply, backward (both gradients in one pass).
 * [OPT] _rw_bwd_x_core, _rw_bwd_probs_core, _RouterWeightMulFunction.backward:
 *   grad_x[r, h]  = (g[r, h].float() * probs[r]).to(x_dt)         (bitwise)
 *   grad_probs[r] = sum_h g[r, h].float() * x[r, h].float()       (fp32)
 * grad_out    g_dt [rows, hidden] contiguous (the forward output's dtype)
 * x           x_dt [rows, hidden] contiguous, or NULL when the forward did
 *             not save x (save_x false): then grad_probs must be NULL too and
 *             only grad_x is computed (x is never read).  With hidden == 0, x
 *             has no elements and may be NULL either way.
 * probs       fp32 [rows]
 * grad_x      x_dt [rows, hidden]  (output)
 * grad_probs  fp32 [rows] or NULL  (output; fixed-order row reduction; the
 *             empty sum +0 when hidden == 0)
 * ---------------------------------------------------------------------- */
MOE_API int moe_router_weight_mul_bwd(const void* grad_out, moe_dtype g_dt, const void* x,
                              moe_dtype x_dt, const float* probs, void* grad_x,
                              float* grad_probs, int64_t rows, int64_t hidden,
                              cudaStream_t stream);

/* ------------------------------------------------------------------------
 * The router-weight multiply with routing probabilities of any dtype.
 * [OPT] _rw_fwd_core (probs.float()) and _rw_bwd_probs_core (the sum "cast to
 * probs_dtype"): as moe_router_weight_mul_fwd / _bwd, with probs of dtype
 * probs_dt (bf16, fp16 or fp32; widened exactly to fp32) and grad_probs
 * rounded once (RNE) to probs_dt.  probs and grad_probs are [rows] in
 * probs_dt.  The fp32 entry points above are these with probs_dt = MOE_FP32.
 * ---------------------------------------------------------------------- */
MOE_API int moe_router_weight_mul_fwd_ex(const void* x, moe_dtype x_dt, const void* probs,
                                         moe_dtype probs_dt, void* out, moe_dtype out_dt,
                                         int64_t rows, int64_t hidden, cudaStream_t stream);
MOE_API int moe_router_weight_mul_bwd_ex(const void* grad_out, moe_dtype g_dt, const void* x,
                                         moe_dtype x_dt, const void* probs, moe_dtype probs_dt,
                                         void* grad_x, void* grad_probs, int64_t rows,
                                         int64_t hidden, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Batch-invariant activation with router probabilities over a padded,
 * expert-grouped row layout.
 * [BI] _squared_relu_with_probs_kernel, squared_relu_with_probs,
 *      _swiglu_with_probs_kernel, swiglu_with_probs:
 *   for each row r < *n_used: m = permutation_map[r];
 *     m >= 0: out[r, :] = act(x[r, :]) * probs[m]       (one bf16 rounding,
 *             except SQRELU, whose square is rounded to bf16 first)
 *     m <  0: alignment padding row -- zero-filled if zero_padding, else
 *             left untouched
 *   rows r >= *n_used are neither read nor written.
 *   SQRELU:       out = bf16(bf16(relu(x)^2) * p)
 *   SQRELU_CLAMP: z = clamp_scale * tanh(x / clamp_scale); out = bf16(relu(z)^2 * p)
 *   SWIGLU:       out = bf16(silu(gate) * up * p), gate = x[r, 0:width],
 *                 up = x[r, width:2*width]
 * x                bf16 [max_rows, width] (SWIGLU: [max_rows, 2*width]) contiguous
 * out              bf16 [max_rows, width] contiguous
 * permutation_map  int32 [max_rows] (device): flat index into probs, or < 0
 * n_used           int32 (device): rows in the live, padded prefix
 * probs            fp32 [num_probs] (device), indexed by permutation_map
 * clamp_scale      SQRELU_CLAMP only: finite and > 0 (MOE_ERR_LIMIT otherwise);
 *                  ignored for the other activations
 * dev_err          optional int32 (device): MOE_DEVERR_COUNT, MOE_DEVERR_MAP
 * ---------------------------------------------------------------------- */
MOE_API int moe_act_with_probs_permuted(moe_act act, const void* x, void* out,
                                const int32_t* permutation_map, const int32_t* n_used,
                                const float* probs, int64_t num_probs, int64_t max_rows,
                                int64_t width, float clamp_scale, int zero_padding,
                                int32_t* dev_err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Token-local unpermute that sums expert contributions in a fixed order.
 * [BI] _unpermute_tokens_in_expert_order_kernel, unpermute_tokens_in_expert_order:
 *   for each token t < *valid_tokens:
 *     acc = +0.0f;  for e = 0, 1, ..., E-1 (increasing local expert id):
 *       if inverse_map[t, e] >= 0: acc += expert_output[inverse_map[t, e], :]
 *     out[t, :] = acc rounded once to out_dt
 *   fp32 sequential adds, no atomics; tokens t >= *valid_tokens untouched.
 * expert_output  in_dt [max_rows, hidden] contiguous
 * inverse_map    int32 [tokens, num_local_experts] (device): row or < 0
 * valid_tokens   int32 (device)
 * out            out_dt [tokens, hidden] contiguous
 * num_local_experts  1 .. 4096
 * dev_err        optional int32 (device): MOE_DEVERR_COUNT, MOE_DEVERR_INVERSE
 * ---------------------------------------------------------------------- */
MOE_API int moe_unpermute_ordered(const void* expert_output, moe_dtype in_dt, int64_t max_rows,
                          const int32_t* inverse_map, const int32_t* valid_tokens, void* out,
                          moe_dtype out_dt, int64_t tokens, int64_t hidden,
                          int32_t num_local_experts, int32_t* dev_err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Fused MoE residual add.
 * [RES] module docstring, _moe_residual_add_kernel, fused_moe_residual_add:
 *   out = residual + round_dt(expert_output + shared_expert_output)
 *   each add in fp32, each result rounded to dt: bit-identical to the two
 *   unfused adds.  Reads the three inputs once and writes out once.  The
 *   backward passes grad_out unchanged to all three inputs, so it has no
 *   kernel.
 * all four tensors dt [numel] contiguous, dt in {BF16, FP16, FP32};
 * out may equal residual (in place).
 * ---------------------------------------------------------------------- */
MOE_API int moe_residual_add(const void* expert_output, const void* shared_expert_output,
                     const void* residual, void* out, int64_t numel, moe_dtype dt,
                     cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Device-bounded weighted SwiGLU with routing weights applied at the
 * activation.
 * [BI] _weighted_silu_mul_bounded_kernel, weighted_silu_mul_bounded:
 *   for every flat output element e = r * half_n + j with e < *bound_elems:
 *     out[r, j] = bf16( silu(y[r, j]) * y[r, half_n + j] * weights[r] )
 *   fp32 math, one rounding (the training fused weighted-SwiGLU rounding);
 *   elements at or past the bound are neither read nor written.
 * y             bf16 [rows, 2*half_n] contiguous (gate | up)
 * weights       fp32 [rows] (routing probability of each row, flat)
 * out           bf16 [rows, half_n] contiguous
 * bound_elems   int64 (device): live_rows * half_n in normal use; a value
 *               outside [0, rows*half_n] is clamped and MOE_DEVERR_COUNT set
 * num_programs  persistent CTAs (<= 0: SMs x resident CTAs per SM).  The grid
 *               size cannot change any output bit.
 * dev_err       optional int32 (device)
 * ---------------------------------------------------------------------- */
MOE_API int moe_weighted_silu_mul_bounded(const void* y, const float* weights, void* out,
                                          const int64_t* bound_elems, int64_t rows,
                                          int64_t half_n, int32_t num_programs,
                                          int32_t* dev_err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Fused epilogue chain: router-weight multiply -> fixed-order unpermute ->
 * residual + (routed + shared) add, in one kernel.
 * Composition of [OPT] _rw_fwd_core (per expert-output row, with that row's
 * permuted probability), [BI] _unpermute_tokens_in_expert_order_kernel and
 * [RES] fused_moe_residual_add; bit-identical to
 *   moe_router_weight_mul_fwd(eo rows, dt -> dt)  then
 *   moe_unpermute_ordered(dt -> dt)               then
 *   moe_residual_add(dt)
 * because every rounding of the chain is kept:
 *   for each token t < *valid_tokens:
 *     acc = +0;  for e ascending with row = inverse_map[t, e] >= 0:
 *       acc += round_dt(expert_output[row, :] * row_probs[row])
 *     out[t, :] = round_dt(residual[t, :] + round_dt(round_dt(acc) + shared[t, :]))
 *   tokens t >= *valid_tokens are untouched.  The expert rows, the shared
 *   output and the residual are read once and out is written once; nothing
 *   else touches memory.
 * expert_output  dt [max_rows, hidden] contiguous (expert-grouped FC2 output)
 * row_probs      fp32 [max_rows]: routing probability of each expert-output
 *                row (the permuted probabilities; unread for padding rows)
 * inverse_map    int32 [tokens, num_local_experts] (device): row or < 0
 * valid_tokens   int32 (device)
 * shared_expert_output, residual, out   dt [tokens, hidden] contiguous;
 *                out may equal residual (in place)
 * dt             MOE_BF16, MOE_FP16 or MOE_FP32 (all tensors)
 * dev_err        optional int32 (device): MOE_DEVERR_COUNT, MOE_DEVERR_INVERSE
 * ---------------------------------------------------------------------- */
MOE_API int moe_epilogue_fused(const void* expert_output, const float* row_probs,
                               int64_t max_rows, const int32_t* inverse_map,
                               const int32_t* valid_tokens, const void* shared_expert_output,
                               const void* residual, void* out, int64_t tokens, int64_t hidden,
                               int32_t num_local_experts, moe_dtype dt, int32_t* dev_err,
                               cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Rank-order reduce-scatter of variable token rows.
 * [BI] ordered_reduce_scatter_v, _ordered_reduce_scatter_v_kernel (reduce
 * peer rows with an explicit rank-order fp32 sum).  Every rank q holds at
 * buffers[q] + input_byte_offset a row-major [capacity_rows, hidden] block
 * (in_dt) of partial results for the tokens of all ranks; rank q's tokens are
 * the rows starting at rank_token_offset[q].  This call writes this rank's
 *   out[t, h] = out_dt( ((x_0 + x_1) + ...) + x_{world-1} ),
 *   x_q = f32(input_q[rank_token_offset[rank] + t, h]),  t < local_tokens,
 * each add in fp32 in rank order and one rounding, so the bits depend on
 * nothing but the inputs.  Only the first *ep_tokens rows of each block hold
 * data (the page's ep_max_tokens): an *ep_tokens outside [0, capacity_rows]
 * is clamped, and an output row whose source row lies outside the data is
 * neither read nor written; both set MOE_DEVERR_COUNT.
 * buffers            DEVICE array of `world` pointers, rank order, each
 *                    addressable from this GPU: its own memory, or a peer's
 *                    mapped into this process (moe_ipc_open).  Read with plain
 *                    loads (no bulk copies, no multicast).
 * input_byte_offset  >= 0, a multiple of in_dt's size
 * world              1..64;  rank in [0, world)
 * rank_token_offset  int32 [world] (device)
 * ep_tokens          int32 (device)
 * out                out_dt [local_tokens, hidden] contiguous, this GPU
 * dev_err            optional int32 (device)
 * Ordering is the caller's: the launch must follow the completion of every
 * rank's input block, and no rank may overwrite its block until every rank's
 * launch has completed (e.g. a stream-ordered barrier -- a one-element
 * all-reduce -- before and after).  The kernel waits on nothing.  Fast path:
 * hidden % 8 == 0, out, input_byte_offset and every buffer 16-byte aligned.
 * ---------------------------------------------------------------------- */
MOE_API int moe_ordered_reduce_scatter_v(const void* const* buffers, int64_t input_byte_offset,
                                         int32_t world, int32_t rank,
                                         const int32_t* rank_token_offset,
                                         const int32_t* ep_tokens, int64_t capacity_rows,
                                         void* out, int64_t local_tokens, int64_t hidden,
                                         moe_dtype in_dt, moe_dtype out_dt, int32_t* dev_err,
                                         cudaStream_t stream);

/* ------------------------------------------------------------------------
 * EP combine: every rank's fixed-order unpermute and the rank-order
 * reduce-scatter of the results, in one kernel over peer memory.
 * [BI] _unpermute_tokens_in_expert_order_kernel followed by
 * ordered_reduce_scatter_v, with the same bits as running them one after the
 * other through blocks of partial sums of dtype partial_dt -- but no partial
 * block is written or read:
 *   for t < local_tokens, g = rank_token_offset[rank] + t:
 *     for q = 0 .. world-1 (rank order):
 *       part_q = partial_dt( +0 + sum over e ascending, row = inverse_maps[q][g, e]
 *                            >= 0, of f32(expert_outputs[q][row, :]) )
 *       acc = (q == 0) ? part_q : acc + part_q                          (fp32)
 *     out[t, :] = out_dt(acc)
 * expert_outputs     DEVICE array of `world` pointers (rank order) to each
 *                    rank's expert-grouped rows, eo_dt [max_rows, hidden]
 *                    contiguous, addressable from this GPU (own memory, or a
 *                    peer's mapped with moe_ipc_open); read with 1-D bulk copies
 *                    into shared memory (16-byte aligned bases, hidden % 8 == 0,
 *                    up to 64 (rank, local expert) pairs) or plain loads, never
 *                    with multicast
 * inverse_maps       DEVICE array of `world` pointers to each rank's int32
 *                    [capacity_rows, num_local_experts] inverse map over the
 *                    token rows of all ranks (row in that rank's expert
 *                    outputs, or < 0); num_local_experts <= 64
 * ep_tokens          int32 (device): token rows that hold data (the pages'
 *                    ep_max_tokens); clamped to capacity_rows
 * world <= 64, rank, rank_token_offset int32 [world] (device): as for
 *                    moe_ordered_reduce_scatter_v
 * partial_dt         the partial blocks' dtype: eo_dt or MOE_FP32
 * out                out_dt [local_tokens, hidden] contiguous; out_dt is eo_dt
 *                    or MOE_FP32
 * dev_err            optional int32 (device): MOE_DEVERR_COUNT (rows outside
 *                    the data: not written), MOE_DEVERR_INVERSE (an entry of
 *                    this rank's tokens >= max_rows: skipped)
 * Ordering is the caller's: the launch must follow the completion of every
 * rank's expert outputs, and no rank may overwrite them until every rank's
 * launch has completed.  The kernel waits on nothing.
 * ---------------------------------------------------------------------- */
MOE_API int moe_unpermute_reduce_scatter(const void* const* expert_outputs, moe_dtype eo_dt,
                                         int64_t max_rows, const int32_t* const* inverse_maps,
                                         int32_t num_local_experts, int64_t capacity_rows,
                                         const int32_t* ep_tokens, int32_t world, int32_t rank,
                                         const int32_t* rank_token_offset, moe_dtype partial_dt,
                                         void* out, moe_dtype out_dt, int64_t local_tokens,
                                         int64_t hidden, int32_t* dev_err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Test hook of the failure path of the bounded waits (no counterpart on the
 * pages; for tests of the error handling, not for production use).
 * The TMA-staged clamped-SwiGLU forward on contiguous x [rows, 2*inter] and
 * y [rows, inter] with `grid` CTAs, except that the copy of row `stall_row`
 * is never issued and its barrier never arrived on: the consumer of that row
 * gives up after `wait_cycles` SM cycles, and so does every warp of its CTA
 * that later waits on it (the producer for a free stage, the other consumers
 * for rows that were never filled).  The CTA then drains its issued copies
 * and exits: no copy is left in flight and no wait is unbounded.  *dev_err
 * receives MOE_DEVERR_TIMEOUT; the other CTAs' rows (r % grid != stall_row %
 * grid) are written as by moe_swiglu_clamped_fwd, row stall_row is not
 * written, and the CUDA context stays usable.
 * dt        MOE_BF16 or MOE_FP16; rows >= 1; inter a multiple of 8, >= 512 and
 *           small enough for the shared-memory ring (MOE_ERR_SHAPE otherwise)
 * grid      1 .. min(rows, SM count);  stall_row in [0, rows)
 * wait_cycles  1000 .. 2^31
 * x, y      16-byte aligned (MOE_ERR_ALIGN);  dev_err required (MOE_ERR_NULL)
 * ---------------------------------------------------------------------- */
MOE_API int moe_test_swiglu_fwd_stalled(const void* x, const float* probs, void* y,
                                        int64_t rows, int64_t inter, float limit, moe_dtype dt,
                                        int32_t grid, int64_t stall_row, int64_t wait_cycles,
                                        int32_t* dev_err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Buffers shared between the processes of one node (CUDA IPC): the plumbing
 * under moe_ordered_reduce_scatter_v's `buffers` (the pages use a symmetric-
 * memory handle; this library maps plain device allocations instead).
 * moe_symm_alloc  cudaMalloc of `bytes` on the current device, zero-filled;
 *                 *ptr owned by the caller, released with moe_symm_free.
 * moe_ipc_export  writes the MOE_IPC_HANDLE_BYTES-byte handle of an allocation
 *                 made by moe_symm_alloc (host memory) for other processes.
 * moe_ipc_open    maps another process's allocation into this one (peer access
 *                 enabled as needed); *ptr is valid until moe_ipc_close.  A
 *                 process cannot open its own handle (MOE_ERR_CUDA).
 * Errors: MOE_ERR_NULL for NULL arguments, MOE_ERR_CUDA with
 * moe_last_cuda_error() set otherwise.
 * ---------------------------------------------------------------------- */
#define MOE_IPC_HANDLE_BYTES 64
MOE_API int moe_symm_alloc(size_t bytes, void** ptr);
MOE_API int moe_symm_free(void* ptr);
MOE_API int moe_ipc_export(const void* ptr, void* handle);
MOE_API int moe_ipc_open(const void* handle, void** ptr);
MOE_API int moe_ipc_close(void* ptr);

#ifdef __cplusplus
}
#endif

#endif /* MOE_EPILOGUE_H */
