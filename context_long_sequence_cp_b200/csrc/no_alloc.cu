// no_alloc.cu — the Ulysses forward that allocates nothing.
//
// For callers that cannot call cudaMalloc when they run attention (their device
// memory belongs to another allocator, or allocation is not allowed where they
// call from), the head-group copies of Q, K, V and O that the Ulysses path
// needs live in one fixed device array owned by this file instead of a
// caller-provided workspace. The array is CP_NOALLOC_SCRATCH_BYTES (32 MiB) and
// exists on every GPU that loads the library's kernels until the process exits.
//
// Host code must not pass `g_noalloc_scratch` itself to a kernel: in host code
// that name is a host-side stand-in, not a device address. The device address
// is looked up once per device with cudaGetSymbolAddress (device current) on
// the first call there, cached, and passed down to the kernels.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "attn_fwd.h"
#include "cp_attn.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[CP_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (first call: look it up).
// The current device must be the plan's: the plan's work list and status word
// live there, and a kernel given another GPU's scratch would read the wrong memory.
int scratch_on_current_device(int plan_device, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CP_ERR_CUDA;
  if (dev != plan_device) return CP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return CP_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return CP_OK;
}

}  // namespace

extern "C" CP_API int cp_attn_fwd_ulysses_noalloc(cp_attn_plan_t plan, const void* q, const void* k,
                                                  const void* v, void* o, float* lse, cp_stream_t stream) {
  if (plan == nullptr) return CP_ERR_INVALID_ARG;
  const size_t need = cp_attn_workspace_bytes(plan, 0);
  if (need == 0) return CP_ERR_UNSUPPORTED;                       // not a Ulysses plan
  if (need > CP_NOALLOC_SCRATCH_BYTES) return CP_ERR_WORKSPACE;   // beyond the fixed scratch
  void* scratch = nullptr;
  const int rc = scratch_on_current_device(cp_internal_plan_device(plan), &scratch);
  if (rc != CP_OK) return rc;
  return cp_internal_ulysses_fwd_scratch(plan, q, k, v, o, lse, scratch, CP_NOALLOC_SCRATCH_BYTES,
                                         static_cast<cudaStream_t>(stream));
}
