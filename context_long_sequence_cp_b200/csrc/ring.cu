// ring.cu — host-side plumbing of the multi-GPU ring: device buffers that other
// ranks' processes can map (CUDA IPC), and the transfer of a peer's key/value
// block into this GPU's memory.
//
// Page "序列与上下文并行", section "上下文并行：注意力本身切分": every rank keeps
// its own Q chunk and receives the K/V blocks of the other ranks one ring step at
// a time, computing on the block it holds while the next one arrives; each step
// moves one rank's K/V. On B200 the block is pulled from the peer's HBM by the
// copy engine (a cudaMemcpyAsync between device pointers over NVLink), so the
// transfer takes no SM away from the persistent attention kernel it overlaps,
// and the attention kernel reads its keys and values from local memory only.
// Ordering between ranks is left to the caller (host-side events and barriers);
// nothing here waits on another GPU.
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
