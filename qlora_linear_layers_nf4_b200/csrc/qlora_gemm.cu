// QLoRA linear forward / backward launchers (tensor-core path in progress).
#include "nf4_common.cuh"
#include "kernels.h"

namespace nf4 {

size_t linear_workspace_bytes(bool, int64_t, int64_t, int64_t, int) { return 0; }

cudaError_t launch_linear_fwd(const LinearArgs&, int, cudaStream_t, int*) {
  return cudaErrorNotSupported;
}

cudaError_t launch_linear_bwd(const LinearArgs&, int, cudaStream_t, int*) {
  return cudaErrorNotSupported;
}

}  // namespace nf4
