// ring.cu — host-side plumbing of the multi-GPU ring: device buffers that other
// ranks' processes can map (CUDA IPC), and a device-to-device copy.
//
// Page "序列与上下文并行", section "上下文并行：注意力本身切分": every rank keeps
// its own Q chunk and receives the K/V blocks of the other ranks, computing on
// the blocks it holds while the next ones arrive. Each rank exposes its own block
// in a slot buffer allocated here; the other ranks map it through CUDA IPC and
// the copy warps of their one-launch ring forward read it over NVLink into local
// slots (attn_fwd.cu). cp_copy_async is a plain cudaMemcpyAsync (the driver's own
// fill of the local slot, and the per-step primitive's callers); such a copy can
// need SM time, so no kernel waits for one. Nothing here waits on another GPU.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "cp_attn.h"

extern "C" {

int cp_ring_buffer_alloc(size_t bytes, void** out) {
  if (out == nullptr) return CP_ERR_INVALID_ARG;
  *out = nullptr;
  if (bytes == 0) return CP_ERR_INVALID_ARG;
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) {
    cudaGetLastError();
    return CP_ERR_CUDA;
  }
  *out = p;
  return CP_OK;
}

int cp_ring_buffer_free(void* p) {
  if (p == nullptr) return CP_OK;
  return cudaFree(p) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

int cp_ipc_handle_bytes(void) { return static_cast<int>(sizeof(cudaIpcMemHandle_t)); }

int cp_ipc_get_handle(const void* base, void* handle_out) {
  if (base == nullptr || handle_out == nullptr) return CP_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, const_cast<void*>(base)) != cudaSuccess) {
    cudaGetLastError();
    return CP_ERR_CUDA;
  }
  std::memcpy(handle_out, &h, sizeof(h));
  return CP_OK;
}

int cp_ipc_open_handle(const void* handle, void** base_out) {
  if (handle == nullptr || base_out == nullptr) return CP_ERR_INVALID_ARG;
  *base_out = nullptr;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    return CP_ERR_CUDA;
  }
  *base_out = p;
  return CP_OK;
}

int cp_ipc_close_handle(void* base) {
  if (base == nullptr) return CP_OK;
  return cudaIpcCloseMemHandle(base) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

int cp_copy_async(void* dst, const void* src, size_t bytes, cp_stream_t stream) {
  if (bytes == 0) return CP_OK;
  if (dst == nullptr || src == nullptr) return CP_ERR_INVALID_ARG;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? CP_OK
             : CP_ERR_CUDA;
}

}  // extern "C"
