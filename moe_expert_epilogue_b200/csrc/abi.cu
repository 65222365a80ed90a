// abi.cu -- the C entry points: argument validation (before anything touches
// the device), persistent-grid sizing, and the status strings.
//
// Validation mirrors the capability predicates of the pages
// (nemo_automodel.components.moe.swiglu_triton.uses_triton_kernel: a 2-D
// row-major x with one probability per row;
// core.fusions.fused_moe_residual_add.can_use_fused_moe_residual_add: same
// shape and dtype in {BF16, FP16, FP32}) and the swiglu_limit > 0 contract of
// the clamped SwiGLU.  Sizes of zero return MOE_OK without a launch; the one
// output an empty size still defines, a probability-gradient sum over no
// terms, is written as +0 by a memset.
#include <atomic>
#include <cmath>
#include <mutex>
#include <unordered_map>

#include "common.cuh"
#include "launch.cuh"
#include "tma.cuh"

namespace moe {

namespace {

thread_local int g_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];

// Resident CTAs per SM by (kernel, dynamic shared memory, device): the same
// kernel launched with more shared memory may fit fewer CTAs on an SM.
struct OccKey {
  const void* kernel;
  size_t smem;
  int device;
  bool operator==(const OccKey& o) const {
    return kernel == o.kernel && smem == o.smem && device == o.device;
  }
};
struct OccKeyHash {
  size_t operator()(const OccKey& k) const {
    size_t h = std::hash<const void*>()(k.kernel);
    h ^= std::hash<size_t>()(k.smem) + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
    h ^= std::hash<int>()(k.device) + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
    return h;
  }
};
std::mutex g_occ_mutex;
std::unordered_map<OccKey, int, OccKeyHash>& occ_cache() {
  static std::unordered_map<OccKey, int, OccKeyHash> m;
  return m;
}

int device_sms(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev >= 0 && dev < kMaxDevices) {
    const int cached = g_sms[dev].load(std::memory_order_relaxed);
    if (cached > 0) { *sms = cached; return MOE_OK; }
  }
  int n = 0;
  e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev >= 0 && dev < kMaxDevices) g_sms[dev].store(n, std::memory_order_relaxed);
  *sms = n;
  return MOE_OK;
}

}  // namespace

int device_sm_count(int* sms) { return device_sms(sms); }

int ensure_smem_limit(const void* kernel, size_t smem) {
  static std::mutex mu;
  static std::unordered_map<const void*, uint64_t> done;  // kernel -> bitmask of devices
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  std::lock_guard<std::mutex> lock(mu);
  if (bit && (done[kernel] & bit)) return MOE_OK;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_fail(e);
  done[kernel] |= bit;
  return MOE_OK;
}

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return MOE_ERR_CUDA;
}

// The sum over no terms is +0: all-zero bits in every dtype of the library.
int zero_fill(void* p, int64_t bytes, cudaStream_t stream) {
  if (!p || bytes <= 0) return MOE_OK;
  const cudaError_t e = cudaMemsetAsync(p, 0, (size_t)bytes, stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

int check_launch() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

int persistent_grid(const void* kernel, size_t smem, int64_t useful_blocks, int* grid) {
  int sms = 0;
  if (int rc = device_sms(&sms)) return rc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  const OccKey key{kernel, smem, dev};
  int per_sm = 0;
  {
    std::lock_guard<std::mutex> lock(g_occ_mutex);
    auto& m = occ_cache();
    auto it = m.find(key);
    if (it != m.end()) {
      per_sm = it->second;
    } else {
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
      if (e != cudaSuccess) return cuda_fail(e);
      if (per_sm < 1) per_sm = 1;
      m.emplace(key, per_sm);
    }
  }
  int64_t g = (int64_t)sms * per_sm;
  if (useful_blocks < g) g = useful_blocks;
  *grid = (int)(g < 1 ? 1 : g);
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

namespace {

inline bool dtype_ok(moe_dtype d) { return d == MOE_BF16 || d == MOE_FP16 || d == MOE_FP32; }
inline int64_t dtype_size(moe_dtype d) { return d == MOE_FP32 ? 4 : 2; }
inline bool aligned_to(const void* p, int64_t n) {
  return (reinterpret_cast<uintptr_t>(p) % (uintptr_t)n) == 0;
}
// rows * cols fits comfortably in int64 element offsets
inline bool product_ok(int64_t a, int64_t b) { return a == 0 || b <= INT64_MAX / 8 / a; }
inline bool limit_ok(float L) { return !std::isnan(L) && L > 0.0f; }

}  // namespace

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_NULL: return "MOE_ERR_NULL: a required pointer is NULL";
    case MOE_ERR_SHAPE: return "MOE_ERR_SHAPE: invalid size or leading dimension";
    case MOE_ERR_DTYPE: return "MOE_ERR_DTYPE: unsupported dtype or activation";
    case MOE_ERR_ALIGN: return "MOE_ERR_ALIGN: pointer not aligned to its element size";
    case MOE_ERR_LIMIT: return "MOE_ERR_LIMIT: limit / clamp_scale must be a positive number";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA runtime error (see moe_last_cuda_error)";
    default: return "unknown moe status";
  }
}

int moe_last_cuda_error(void) { return g_last_cuda_error; }

int moe_abi_version(void) { return 1; }

int moe_swiglu_clamped_fwd_ex(const void* x, const float* probs, void* y, int64_t rows,
                              int64_t inter, int64_t ld_x, int64_t ld_y, float limit,
                              moe_dtype dt, int32_t* dev_err, cudaStream_t stream) {
  if (!dtype_ok(dt)) return MOE_ERR_DTYPE;
  if (rows < 0 || inter < 0 || ld_x < 2 * inter || ld_y < inter) return MOE_ERR_SHAPE;
  if (!product_ok(rows, ld_x) || !product_ok(rows, ld_y)) return MOE_ERR_SHAPE;
  if (!limit_ok(limit)) return MOE_ERR_LIMIT;
  if (rows == 0 || inter == 0) return MOE_OK;
  if (!x || !probs || !y) return MOE_ERR_NULL;
  const int64_t es = dtype_size(dt);
  if (!aligned_to(x, es) || !aligned_to(y, es) || !aligned_to(probs, 4) ||
      !aligned_to(dev_err, 4))
    return MOE_ERR_ALIGN;
  return launch_swiglu_clamped_fwd(x, probs, y, rows, inter, ld_x, ld_y, limit, dt, dev_err,
                                   stream);
}

int moe_swiglu_clamped_fwd(const void* x, const float* probs, void* y, int64_t rows,
                           int64_t inter, int64_t ld_x, int64_t ld_y, float limit,
                           moe_dtype dt, cudaStream_t stream) {
  return moe_swiglu_clamped_fwd_ex(x, probs, y, rows, inter, ld_x, ld_y, limit, dt, nullptr,
                                   stream);
}

int moe_test_swiglu_fwd_stalled(const void* x, const float* probs, void* y, int64_t rows,
                                int64_t inter, float limit, moe_dtype dt, int32_t grid,
                                int64_t stall_row, int64_t wait_cycles, int32_t* dev_err,
                                cudaStream_t stream) {
  if (dt != MOE_BF16 && dt != MOE_FP16) return MOE_ERR_DTYPE;
  int sms = 0;
  if (int rc = device_sm_count(&sms)) return rc;
  if (rows < 1 || !product_ok(rows, 2 * inter) || !tma_forward_applies(inter, dt) ||
      grid < 1 || grid > sms || (int64_t)grid > rows || stall_row < 0 || stall_row >= rows ||
      wait_cycles < 1000 || wait_cycles > tma::kWaitCycles)
    return MOE_ERR_SHAPE;
  if (!limit_ok(limit)) return MOE_ERR_LIMIT;
  if (!x || !probs || !y || !dev_err) return MOE_ERR_NULL;
  if (!aligned_to(x, 16) || !aligned_to(y, 16) || !aligned_to(probs, 4) ||
      !aligned_to(dev_err, 4))
    return MOE_ERR_ALIGN;
  return launch_swiglu_fwd_stalled(x, probs, y, rows, inter, limit, dt, grid, stall_row,
                                   (long long)wait_cycles, dev_err, stream);
}

int moe_swiglu_clamped_bwd(const void* x, const float* probs, const void* grad_y,
                           void* grad_x, float* grad_probs, int64_t rows, int64_t inter,
                           int64_t ld_x, int64_t ld_gy, int64_t ld_gx, float limit,
                           moe_dtype dt, cudaStream_t stream) {
  if (!dtype_ok(dt)) return MOE_ERR_DTYPE;
  if (rows < 0 || inter < 0 || ld_x < 2 * inter || ld_gy < inter || ld_gx < 2 * inter)
    return MOE_ERR_SHAPE;
  if (!product_ok(rows, ld_x) || !product_ok(rows, ld_gy) || !product_ok(rows, ld_gx))
    return MOE_ERR_SHAPE;
  if (!limit_ok(limit)) return MOE_ERR_LIMIT;
  if (rows == 0) return MOE_OK;
  if (!probs || !grad_probs) return MOE_ERR_NULL;
  if (inter > 0 && (!x || !grad_y || !grad_x)) return MOE_ERR_NULL;
  const int64_t es = dtype_size(dt);
  if (!aligned_to(x, es) || !aligned_to(grad_y, es) || !aligned_to(grad_x, es) ||
      !aligned_to(probs, 4) || !aligned_to(grad_probs, 4))
    return MOE_ERR_ALIGN;
  if (inter == 0) return zero_fill(grad_probs, rows * 4, stream);   // empty sums: +0
  return launch_swiglu_clamped_bwd(x, probs, grad_y, grad_x, grad_probs, rows, inter, ld_x,
                                   ld_gy, ld_gx, limit, dt, stream);
}

int moe_router_weight_mul_fwd_ex(const void* x, moe_dtype x_dt, const void* probs,
                                 moe_dtype probs_dt, void* out, moe_dtype out_dt, int64_t rows,
                                 int64_t hidden, cudaStream_t stream) {
  if (!dtype_ok(x_dt) || !dtype_ok(out_dt) || !dtype_ok(probs_dt)) return MOE_ERR_DTYPE;
  if (rows < 0 || hidden < 0 || !product_ok(rows, hidden)) return MOE_ERR_SHAPE;
  if (rows == 0 || hidden == 0) return MOE_OK;
  if (!x || !probs || !out) return MOE_ERR_NULL;
  if (!aligned_to(x, dtype_size(x_dt)) || !aligned_to(out, dtype_size(out_dt)) ||
      !aligned_to(probs, dtype_size(probs_dt)))
    return MOE_ERR_ALIGN;
  return launch_router_weight_fwd(x, x_dt, probs, probs_dt, out, out_dt, rows, hidden, stream);
}

int moe_router_weight_mul_fwd(const void* x, moe_dtype x_dt, const float* probs, void* out,
                              moe_dtype out_dt, int64_t rows, int64_t hidden,
                              cudaStream_t stream) {
  return moe_router_weight_mul_fwd_ex(x, x_dt, probs, MOE_FP32, out, out_dt, rows, hidden,
                                      stream);
}

int moe_router_weight_mul_bwd_ex(const void* grad_out, moe_dtype g_dt, const void* x,
                                 moe_dtype x_dt, const void* probs, moe_dtype probs_dt,
                                 void* grad_x, void* grad_probs, int64_t rows, int64_t hidden,
                                 cudaStream_t stream) {
  if (!dtype_ok(g_dt) || !dtype_ok(x_dt) || !dtype_ok(probs_dt)) return MOE_ERR_DTYPE;
  if (rows < 0 || hidden < 0 || !product_ok(rows, hidden)) return MOE_ERR_SHAPE;
  // x and grad_probs come together (save_x); with hidden == 0 x has no
  // elements and may be NULL, and grad_probs alone asks for the empty sums.
  if (hidden > 0 && (x == nullptr) != (grad_probs == nullptr)) return MOE_ERR_NULL;
  if (rows == 0) return MOE_OK;
  if (!probs) return MOE_ERR_NULL;
  if (hidden > 0 && (!grad_out || !grad_x)) return MOE_ERR_NULL;
  if (!aligned_to(grad_out, dtype_size(g_dt)) || !aligned_to(x, dtype_size(x_dt)) ||
      !aligned_to(grad_x, dtype_size(x_dt)) || !aligned_to(probs, dtype_size(probs_dt)) ||
      !aligned_to(grad_probs, dtype_size(probs_dt)))
    return MOE_ERR_ALIGN;
  if (hidden == 0) return zero_fill(grad_probs, rows * dtype_size(probs_dt), stream);
  return launch_router_weight_bwd(grad_out, g_dt, x, x_dt, probs, probs_dt, grad_x, grad_probs,
                                  rows, hidden, stream);
}

int moe_router_weight_mul_bwd(const void* grad_out, moe_dtype g_dt, const void* x,
                              moe_dtype x_dt, const float* probs, void* grad_x,
                              float* grad_probs, int64_t rows, int64_t hidden,
                              cudaStream_t stream) {
  return moe_router_weight_mul_bwd_ex(grad_out, g_dt, x, x_dt, probs, MOE_FP32, grad_x,
                                      grad_probs, rows, hidden, stream);
}

int moe_act_with_probs_permuted(moe_act act, const void* x, void* out,
                                const int32_t* permutation_map, const int32_t* n_used,
                                const float* probs, int64_t num_probs, int64_t max_rows,
                                int64_t width, float clamp_scale, int zero_padding,
                                int32_t* dev_err, cudaStream_t stream) {
  if (act != MOE_ACT_SQRELU && act != MOE_ACT_SQRELU_CLAMP && act != MOE_ACT_SWIGLU)
    return MOE_ERR_DTYPE;
  if (num_probs < 0 || max_rows < 0 || width < 0 || max_rows > INT32_MAX ||
      !product_ok(max_rows, 2 * width))
    return MOE_ERR_SHAPE;
  if (act == MOE_ACT_SQRELU_CLAMP && !(std::isfinite(clamp_scale) && clamp_scale > 0.0f))
    return MOE_ERR_LIMIT;
  if (max_rows == 0 || width == 0) return MOE_OK;
  if (!x || !out || !permutation_map || !n_used || (num_probs > 0 && !probs))
    return MOE_ERR_NULL;
  if (!aligned_to(x, 2) || !aligned_to(out, 2) || !aligned_to(permutation_map, 4) ||
      !aligned_to(n_used, 4) || !aligned_to(probs, 4) || !aligned_to(dev_err, 4))
    return MOE_ERR_ALIGN;
  return launch_act_with_probs_permuted(act, static_cast<const uint16_t*>(x),
                                        static_cast<uint16_t*>(out), permutation_map, n_used,
                                        probs, num_probs, max_rows, width, clamp_scale,
                                        zero_padding, dev_err, stream);
}

int moe_unpermute_ordered(const void* expert_output, moe_dtype in_dt, int64_t max_rows,
                          const int32_t* inverse_map, const int32_t* valid_tokens, void* out,
                          moe_dtype out_dt, int64_t tokens, int64_t hidden,
                          int32_t num_local_experts, int32_t* dev_err, cudaStream_t stream) {
  if (!dtype_ok(in_dt) || !dtype_ok(out_dt)) return MOE_ERR_DTYPE;
  if (max_rows < 0 || tokens < 0 || hidden < 0 || num_local_experts < 1 ||
      num_local_experts > 4096 || max_rows > INT32_MAX || !product_ok(max_rows, hidden) ||
      !product_ok(tokens, hidden) || !product_ok(tokens, num_local_experts))
    return MOE_ERR_SHAPE;
  if (tokens == 0 || hidden == 0) return MOE_OK;
  if (!inverse_map || !valid_tokens || !out || (max_rows > 0 && !expert_output))
    return MOE_ERR_NULL;
  if (!aligned_to(expert_output, dtype_size(in_dt)) || !aligned_to(out, dtype_size(out_dt)) ||
      !aligned_to(inverse_map, 4) || !aligned_to(valid_tokens, 4) || !aligned_to(dev_err, 4))
    return MOE_ERR_ALIGN;
  return launch_unpermute_ordered(expert_output, in_dt, max_rows, inverse_map, valid_tokens, out,
                                  out_dt, tokens, hidden, num_local_experts, dev_err, stream);
}

int moe_residual_add(const void* expert_output, const void* shared_expert_output,
                     const void* residual, void* out, int64_t numel, moe_dtype dt,
                     cudaStream_t stream) {
  if (!dtype_ok(dt)) return MOE_ERR_DTYPE;
  if (numel < 0 || numel > INT64_MAX / 8) return MOE_ERR_SHAPE;
  if (numel == 0) return MOE_OK;
  if (!expert_output || !shared_expert_output || !residual || !out) return MOE_ERR_NULL;
  const int64_t es = dtype_size(dt);
  if (!aligned_to(expert_output, es) || !aligned_to(shared_expert_output, es) ||
      !aligned_to(residual, es) || !aligned_to(out, es))
    return MOE_ERR_ALIGN;
  return launch_residual_add(expert_output, shared_expert_output, residual, out, numel, dt,
                             stream);
}

int moe_weighted_silu_mul_bounded(const void* y, const float* weights, void* out,
                                  const int64_t* bound_elems, int64_t rows, int64_t half_n,
                                  int32_t num_programs, int32_t* dev_err, cudaStream_t stream) {
  if (rows < 0 || half_n < 0 || !product_ok(rows, 2 * half_n)) return MOE_ERR_SHAPE;
  if (rows == 0 || half_n == 0) return MOE_OK;
  if (!y || !weights || !out || !bound_elems) return MOE_ERR_NULL;
  if (!aligned_to(y, 2) || !aligned_to(out, 2) || !aligned_to(weights, 4) ||
      !aligned_to(bound_elems, 8) || !aligned_to(dev_err, 4))
    return MOE_ERR_ALIGN;
  return launch_weighted_silu_mul_bounded(static_cast<const uint16_t*>(y), weights,
                                          static_cast<uint16_t*>(out), bound_elems, rows, half_n,
                                          num_programs, dev_err, stream);
}

int moe_epilogue_fused(const void* expert_output, const float* row_probs, int64_t max_rows,
                       const int32_t* inverse_map, const int32_t* valid_tokens,
                       const void* shared_expert_output, const void* residual, void* out,
                       int64_t tokens, int64_t hidden, int32_t num_local_experts, moe_dtype dt,
                       int32_t* dev_err, cudaStream_t stream) {
  if (!dtype_ok(dt)) return MOE_ERR_DTYPE;
  if (max_rows < 0 || tokens < 0 || hidden < 0 || num_local_experts < 1 ||
      num_local_experts > 4096 || max_rows > INT32_MAX || !product_ok(max_rows, hidden) ||
      !product_ok(tokens, hidden) || !product_ok(tokens, num_local_experts))
    return MOE_ERR_SHAPE;
  if (tokens == 0 || hidden == 0) return MOE_OK;
  if (!inverse_map || !valid_tokens || !shared_expert_output || !residual || !out ||
      (max_rows > 0 && (!expert_output || !row_probs)))
    return MOE_ERR_NULL;
  const int64_t es = dtype_size(dt);
  if (!aligned_to(expert_output, es) || !aligned_to(shared_expert_output, es) ||
      !aligned_to(residual, es) || !aligned_to(out, es) || !aligned_to(row_probs, 4) ||
      !aligned_to(inverse_map, 4) || !aligned_to(valid_tokens, 4) || !aligned_to(dev_err, 4))
    return MOE_ERR_ALIGN;
  return launch_epilogue_fused(expert_output, row_probs, max_rows, inverse_map, valid_tokens,
                               shared_expert_output, residual, out, tokens, hidden,
                               num_local_experts, dt, dev_err, stream);
}

int moe_ordered_reduce_scatter_v(const void* const* buffers, int64_t input_byte_offset,
                                 int32_t world, int32_t rank, const int32_t* rank_token_offset,
                                 const int32_t* ep_tokens, int64_t capacity_rows, void* out,
                                 int64_t local_tokens, int64_t hidden, moe_dtype in_dt,
                                 moe_dtype out_dt, int32_t* dev_err, cudaStream_t stream) {
  if (!dtype_ok(in_dt) || !dtype_ok(out_dt)) return MOE_ERR_DTYPE;
  if (world < 1 || world > max_reduce_scatter_world() || rank < 0 || rank >= world ||
      local_tokens < 0 || hidden < 0 || capacity_rows < 0 || input_byte_offset < 0 ||
      !product_ok(local_tokens, hidden) || !product_ok(capacity_rows, hidden))
    return MOE_ERR_SHAPE;
  if (local_tokens == 0 || hidden == 0) return MOE_OK;
  if (!buffers || !rank_token_offset || !ep_tokens || !out) return MOE_ERR_NULL;
  if (!aligned_to(buffers, sizeof(void*)) || !aligned_to(rank_token_offset, 4) ||
      !aligned_to(ep_tokens, 4) || !aligned_to(out, dtype_size(out_dt)) ||
      !aligned_to(dev_err, 4) || input_byte_offset % dtype_size(in_dt) != 0)
    return MOE_ERR_ALIGN;
  return launch_ordered_reduce_scatter_v(buffers, input_byte_offset, world, rank,
                                         rank_token_offset, ep_tokens, capacity_rows, out,
                                         local_tokens, hidden, in_dt, out_dt, dev_err, stream);
}

int moe_unpermute_reduce_scatter(const void* const* expert_outputs, moe_dtype eo_dt,
                                 int64_t max_rows, const int32_t* const* inverse_maps,
                                 int32_t num_local_experts, int64_t capacity_rows,
                                 const int32_t* ep_tokens, int32_t world, int32_t rank,
                                 const int32_t* rank_token_offset, moe_dtype partial_dt,
                                 void* out, moe_dtype out_dt, int64_t local_tokens,
                                 int64_t hidden, int32_t* dev_err, cudaStream_t stream) {
  if (!dtype_ok(eo_dt) || !dtype_ok(partial_dt) || !dtype_ok(out_dt)) return MOE_ERR_DTYPE;
  if ((partial_dt != eo_dt && partial_dt != MOE_FP32) || (out_dt != eo_dt && out_dt != MOE_FP32))
    return MOE_ERR_DTYPE;
  if (world < 1 || world > max_ep_combine_world() || rank < 0 || rank >= world ||
      num_local_experts < 1 || num_local_experts > max_ep_combine_experts() || max_rows < 0 ||
      max_rows > INT32_MAX || capacity_rows < 0 || local_tokens < 0 || hidden < 0 ||
      !product_ok(max_rows, hidden) || !product_ok(local_tokens, hidden) ||
      !product_ok(capacity_rows, num_local_experts))
    return MOE_ERR_SHAPE;
  if (local_tokens == 0 || hidden == 0) return MOE_OK;
  if (!expert_outputs || !inverse_maps || !ep_tokens || !rank_token_offset || !out)
    return MOE_ERR_NULL;
  if (!aligned_to(expert_outputs, sizeof(void*)) || !aligned_to(inverse_maps, sizeof(void*)) ||
      !aligned_to(ep_tokens, 4) || !aligned_to(rank_token_offset, 4) ||
      !aligned_to(out, dtype_size(out_dt)) || !aligned_to(dev_err, 4))
    return MOE_ERR_ALIGN;
  return launch_unpermute_reduce_scatter(
      expert_outputs, eo_dt, max_rows, reinterpret_cast<const void* const*>(inverse_maps),
      num_local_experts, capacity_rows, ep_tokens, world, rank, rank_token_offset, partial_dt,
      out, out_dt, local_tokens, hidden, dev_err, stream);
}

}  // extern "C"
