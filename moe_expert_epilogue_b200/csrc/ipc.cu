// ipc.cu -- device buffers shared between the processes of one node.
//
// The rank-order reduce-scatter reads every rank's block of partial results
// through a table of pointers that this GPU can address.  The pages obtain
// that table from a symmetric-memory handle; here each rank allocates a plain
// device buffer, exports its CUDA IPC handle, and maps the other ranks'
// buffers into its own address space (peer access over NVLink is enabled by
// the runtime as the mapping is opened).  Host code only; no kernel here.
#include <cstring>

#include "common.cuh"
#include "launch.cuh"

static_assert(sizeof(cudaIpcMemHandle_t) == MOE_IPC_HANDLE_BYTES,
              "CUDA IPC handle size differs from MOE_IPC_HANDLE_BYTES");

extern "C" {

int moe_symm_alloc(size_t bytes, void** ptr) {
  if (!ptr) return MOE_ERR_NULL;
  *ptr = nullptr;
  if (bytes == 0) return MOE_ERR_SHAPE;
  void* p = nullptr;
  cudaError_t e = cudaMalloc(&p, bytes);
  if (e != cudaSuccess) return moe::cuda_fail(e);
  e = cudaMemset(p, 0, bytes);
  if (e != cudaSuccess) {
    cudaFree(p);
    return moe::cuda_fail(e);
  }
  *ptr = p;
  return MOE_OK;
}

int moe_symm_free(void* ptr) {
  if (!ptr) return MOE_OK;
  cudaError_t e = cudaFree(ptr);
  return e == cudaSuccess ? MOE_OK : moe::cuda_fail(e);
}

int moe_ipc_export(const void* ptr, void* handle) {
  if (!ptr || !handle) return MOE_ERR_NULL;
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, const_cast<void*>(ptr));
  if (e != cudaSuccess) return moe::cuda_fail(e);
  std::memcpy(handle, &h, sizeof(h));
  return MOE_OK;
}

int moe_ipc_open(const void* handle, void** ptr) {
  if (!handle || !ptr) return MOE_ERR_NULL;
  *ptr = nullptr;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* p = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return moe::cuda_fail(e);
  *ptr = p;
  return MOE_OK;
}

int moe_ipc_close(void* ptr) {
  if (!ptr) return MOE_ERR_NULL;
  cudaError_t e = cudaIpcCloseMemHandle(ptr);
  return e == cudaSuccess ? MOE_OK : moe::cuda_fail(e);
}

}  // extern "C"
