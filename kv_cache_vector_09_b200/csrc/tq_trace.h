// NVTX ranges around the library's entry points, so that profilers (Nsight
// Compute's --nvtx filters, Nsight Systems timelines) can attribute kernels to
// the C-ABI call that launched them.  NVTX3 is header-only: with no tool
// attached, a range costs a check of a function pointer.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace tqtrace {

struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

}  // namespace tqtrace
