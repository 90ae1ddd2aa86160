// An NVTX range around one C-ABI call, named after the call, so that a
// profiler's timeline (Nsight Systems) and ncu's NVTX filters show which
// library call enqueued which kernels.  NVTX3 is header-only: with no tool
// attached a range costs a couple of branches and loads nothing.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace nf4 {

struct ApiRange {
  explicit ApiRange(const char* name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
  ApiRange(const ApiRange&) = delete;
  ApiRange& operator=(const ApiRange&) = delete;
};

}  // namespace nf4

#define NF4_API_RANGE(name) const ::nf4::ApiRange nf4_api_range_(name)
