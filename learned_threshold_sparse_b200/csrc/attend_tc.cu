// Tensor-core (tcgen05) attention over the admitted blocks: not built yet;
// every shape reports unsupported and the CUDA-core kernel is used.
#include "eta_internal.h"

namespace eta {

bool attend_tc_supported(const Shape&) { return false; }
size_t attend_tc_smem(const Shape&) { return 0; }
cudaError_t launch_attend_tc(const AttendArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace eta
