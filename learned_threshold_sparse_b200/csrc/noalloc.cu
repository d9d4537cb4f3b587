// eta_decode_noalloc: the decode step for callers that cannot allocate device
// memory, with its scratch in a fixed-size array that the library declares.
//
// eta_decode needs a caller-provided workspace.  Some callers cannot make one:
// a plugin that runs inside a host program which owns every device
// allocation, or a code path where a cudaMalloc would synchronise the whole
// device.  This variant takes the same parameters but ignores
// params->workspace / workspace_bytes and uses g_eta_noalloc_scratch instead.
#include <mutex>

#include "eta_internal.h"

namespace {

// Fixed scratch of every device that loads the library, kept until exit.
constexpr size_t kNoallocScratchBytes = ETA_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_eta_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
eta_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ETA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_eta_noalloc_scratch) != cudaSuccess || p == nullptr) return ETA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ETA_OK;
}

}  // namespace

extern "C" eta_status eta_decode_noalloc(const eta_decode_params* p, void* stream) {
  if (!p) return ETA_ERR_INVALID_ARG;
  eta_decode_params q = *p;
  q.workspace = nullptr;
  q.workspace_bytes = 0;
  size_t need = 0;
  eta_status st = eta_decode_workspace_size(&q, &need);
  if (st != ETA_OK) return st;
  if (need > kNoallocScratchBytes) return ETA_ERR_WORKSPACE;  // shapes too large for the fixed scratch
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != ETA_OK) return st;
  // The previous call's device status word is cleared; everything else the
  // step reads is rewritten by the step itself (the rescue counters are
  // zeroed inside eta_decode when that mode is on).
  if (cudaMemsetAsync(scratch, 0, 16, static_cast<cudaStream_t>(stream)) != cudaSuccess) return ETA_ERR_CUDA;
  q.workspace = scratch;
  q.workspace_bytes = kNoallocScratchBytes;
  return eta_decode(&q, stream);
}
