// eta_decode_noalloc: the decode step for callers that cannot allocate device
// memory, with its scratch in a fixed-size array that the library declares.
//
// eta_decode needs a caller-provided workspace.  Some callers cannot make one:
// a plugin that runs inside a host program which owns every device
// allocation, or a code path where a cudaMalloc would synchronise the whole
// device.  This variant takes the same parameters but ignores
// params->workspace / workspace_bytes and uses g_eta_noalloc_scratch instead.
#include "eta_internal.h"

namespace {

// Fixed scratch of every device that loads the library, kept until exit.
constexpr size_t kNoallocScratchBytes = ETA_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_eta_noalloc_scratch[kNoallocScratchBytes];

// Device address of the scratch array in the current device's context.  In
// host code the array's name is only a host-side stand-in, so the address is
// looked up with that device current.  It is looked up on every call rather
// than cached: after a context reset a cached address would point into a
// context that no longer exists.  The lookup does not touch any stream.
eta_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_eta_noalloc_scratch) != cudaSuccess || p == nullptr) return ETA_ERR_CUDA;
  *out = p;
  return ETA_OK;
}

}  // namespace

extern "C" eta_status eta_decode_noalloc(const eta_decode_params* p, unsigned* device_status, void* stream) {
  if (!p) return ETA_ERR_INVALID_ARG;
  if (device_status && (reinterpret_cast<uintptr_t>(device_status) % 4) != 0) return ETA_ERR_INVALID_ARG;
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
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // The previous call's device status word is cleared; everything else the
  // step reads is rewritten by the step itself (the rescue counters are
  // zeroed inside eta_decode when that mode is on).
  if (cudaMemsetAsync(scratch, 0, 16, cs) != cudaSuccess) return ETA_ERR_CUDA;
  q.workspace = scratch;
  q.workspace_bytes = kNoallocScratchBytes;
  st = eta_decode(&q, stream);
  if (st != ETA_OK) return st;
  // The step's status word, handed to the caller's device word (stream-ordered).
  if (device_status &&
      cudaMemcpyAsync(device_status, scratch, sizeof(unsigned), cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
    return ETA_ERR_CUDA;
  return ETA_OK;
}
