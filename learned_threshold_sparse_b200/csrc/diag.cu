// eta_diag_wait_timeout: drives the library's bounded device-side wait to its
// limit on purpose, so that the failure-reporting path (status bit in the
// workspace, ETA_ERR_DEVICE_TIMEOUT from eta_read_device_status, a context
// that stays usable) can be checked end to end without any fault or hang.
// One warp initialises an mbarrier in shared memory that nothing ever
// completes and waits on its first phase with the same helper the kernels
// use; the wait gives up after its cycle limit (about one second) and sets
// the timeout bit.
#include "eta_device.cuh"

namespace {

__global__ void __launch_bounds__(32) diag_wait_kernel(unsigned* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    eta::dev::mbar_init(&bar, 1);
    eta::dev::fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) (void)eta::dev::mbar_wait(&bar, 0, status);  // no arrival: gives up
}

}  // namespace

extern "C" eta_status eta_diag_wait_timeout(void* workspace, void* stream) {
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return ETA_ERR_INVALID_ARG;
  diag_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<unsigned*>(workspace));
  return cudaGetLastError() == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}
