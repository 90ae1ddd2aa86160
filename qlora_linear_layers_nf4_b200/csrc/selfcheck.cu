// Self-check of the bounded-wait path (no counterpart on the pages).
//
// Every mbarrier wait in the library's kernels gives up after a time limit,
// records NF4_ERR_TIMEOUT in the caller's status word, raises its CTA's abort
// flag and lets the kernel unwind, so a lost arrival can never hang the GPU.
// This kernel exercises exactly that path without faulting anything: one warp
// of each CTA waits on a barrier that nothing ever arrives on, with a short
// limit, while a second warp polls the abort flag the way a kernel's other
// roles do; both then return normally.
#include <cuda.h>

#include "kernels.h"
#include "nf4_common.cuh"
#include "tc_common.cuh"

namespace nf4 {
namespace {

using namespace tc;

__global__ void __launch_bounds__(64) wait_timeout_check_kernel(uint32_t* status, uint64_t limit_ns,
                                                                uint32_t* seen_abort) {
  __shared__ uint64_t never;            // a barrier that no thread or copy arrives on
  __shared__ uint64_t other;            // the second role's barrier, also never completed
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);
    mbar_init(&other, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    // waits out the limit, then reports and aborts
    (void)__all_sync(0xffffffffu, mbar_wait_limit(&never, 0, &abort_flag, status, limit_ns));
  } else {
    // a role with a far longer limit that must notice the abort instead
    const bool ok = __all_sync(0xffffffffu,
                               mbar_wait_limit(&other, 0, &abort_flag, status, 100 * limit_ns));
    if (!ok && threadIdx.x == 32 && abort_flag) atomicAdd(seen_abort, 1u);
  }
}

}  // namespace

cudaError_t launch_wait_timeout_check(uint32_t* status, uint64_t limit_ns, uint32_t* seen_abort,
                                      cudaStream_t st, int* launches) {
  wait_timeout_check_kernel<<<2, 64, 0, st>>>(status, limit_ns, seen_abort);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace nf4
