// launch.cuh -- host-side launch helpers shared by the op launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "moe_epilogue.h"

namespace moe {

// Records a failing CUDA call for moe_last_cuda_error() and returns MOE_ERR_CUDA.
int cuda_fail(cudaError_t e);

// Persistent grid for `kernel` launched with kThreads threads and `smem`
// bytes of dynamic shared memory: resident CTAs per SM (occupancy, cached per
// kernel, shared-memory size and device) times the SM count of the current
// device (cached per device), but no more than `useful_blocks`, and at least 1.
int persistent_grid(const void* kernel, size_t smem, int64_t useful_blocks, int* grid);

// MOE_ERR_CUDA if the launch just issued failed.
int check_launch();

// Enqueue kernel<<<grid, kThreads, smem, stream>>>(args...) with programmatic
// stream serialisation allowed (see pdl_prologue); a failure is left in the
// runtime's error state for check_launch().
template <typename... KArgs, typename... Args>
inline void launch_kernel_block(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                                cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = MOE_PDL;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  (void)cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
inline void launch_kernel(void (*kernel)(KArgs...), int grid, size_t smem, cudaStream_t stream,
                          Args... args) {
  launch_kernel_block(kernel, grid, kThreads, smem, stream, args...);
}

// SM count of the current device (cached per device).
int device_sm_count(int* sms);

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
int ensure_smem_limit(const void* kernel, size_t smem);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// Launchers (one per op family); arguments already validated.
int launch_swiglu_clamped_fwd(const void* x, const float* probs, void* y, int64_t rows,
                              int64_t inter, int64_t ld_x, int64_t ld_y, float limit,
                              moe_dtype dt, int32_t* dev_err, cudaStream_t stream);
// 1 if the forward of rows of `inter` columns of dt takes the TMA-staged kernel
// (given contiguous, 16-byte aligned tensors).
int tma_forward_applies(int64_t inter, moe_dtype dt);
// The TMA-staged forward with one row's fill withheld (tests of the bounded
// waits; contiguous x and y, arguments validated by the caller).
int launch_swiglu_fwd_stalled(const void* x, const float* probs, void* y, int64_t rows,
                              int64_t inter, float limit, moe_dtype dt, int grid,
                              int64_t stall_row, long long wait_cycles, int32_t* dev_err,
                              cudaStream_t stream);
int launch_swiglu_clamped_bwd(const void* x, const float* probs, const void* grad_y,
                              void* grad_x, float* grad_probs, int64_t rows, int64_t inter,
                              int64_t ld_x, int64_t ld_gy, int64_t ld_gx, float limit,
                              moe_dtype dt, cudaStream_t stream);
int max_ep_combine_world();
// Copies (and optionally clears) the EP combine's per-device timeout word.
int ep_combine_device_errors(int32_t* bits, int clear);
int max_ep_combine_experts();
int launch_unpermute_reduce_scatter(const void* const* expert_outputs, moe_dtype eo_dt,
                                    int64_t max_rows, const void* const* inverse_maps,
                                    int num_local_experts, int64_t capacity_rows,
                                    const int32_t* ep_tokens, int world, int rank,
                                    const int32_t* rank_token_offset, moe_dtype partial_dt,
                                    void* out, moe_dtype out_dt, int64_t local_tokens,
                                    int64_t hidden, int32_t* err, cudaStream_t stream);
int max_reduce_scatter_world();
int launch_ordered_reduce_scatter_v(const void* const* bufs, int64_t byte_off, int world, int rank,
                                    const int32_t* offs, const int32_t* ep_tokens,
                                    int64_t capacity, void* out, int64_t local, int64_t hidden,
                                    moe_dtype in_dt, moe_dtype out_dt, int32_t* err,
                                    cudaStream_t stream);
int launch_router_weight_fwd(const void* x, moe_dtype x_dt, const void* probs, moe_dtype p_dt,
                             void* out, moe_dtype out_dt, int64_t rows, int64_t hidden,
                             cudaStream_t stream);
int launch_router_weight_bwd(const void* grad_out, moe_dtype g_dt, const void* x,
                             moe_dtype x_dt, const void* probs, moe_dtype p_dt, void* grad_x,
                             void* grad_probs, int64_t rows, int64_t hidden,
                             cudaStream_t stream);
int launch_act_with_probs_permuted(moe_act act, const uint16_t* x, uint16_t* out,
                                   const int32_t* permutation_map, const int32_t* n_used,
                                   const float* probs, int64_t num_probs, int64_t max_rows,
                                   int64_t width, float clamp_scale, int zero_padding,
                                   int32_t* dev_err, cudaStream_t stream);
int launch_unpermute_ordered(const void* expert_output, moe_dtype in_dt, int64_t max_rows,
                             const int32_t* inverse_map, const int32_t* valid_tokens,
                             void* out, moe_dtype out_dt, int64_t tokens, int64_t hidden,
                             int32_t num_local_experts, int32_t* dev_err,
                             cudaStream_t stream);
int launch_weighted_silu_mul_bounded(const uint16_t* y, const float* weights, uint16_t* out,
                                     const int64_t* bound_elems, int64_t rows, int64_t half_n,
                                     int32_t num_programs, int32_t* dev_err,
                                     cudaStream_t stream);
int launch_epilogue_fused(const void* expert_output, const float* row_probs, int64_t max_rows,
                          const int32_t* inverse_map, const int32_t* valid_tokens,
                          const void* shared_expert_output, const void* residual, void* out,
                          int64_t tokens, int64_t hidden, int32_t num_local_experts,
                          moe_dtype dt, int32_t* dev_err, cudaStream_t stream);
int launch_residual_add(const void* e, const void* s, const void* r, void* out, int64_t numel,
                        moe_dtype dt, cudaStream_t stream);

}  // namespace moe
