// NVTX ranges around the library's entry points, so that timelines and
// profiler filters can find the library's launches (for example
// `ncu --nvtx --nvtx-include "attn_bwd/"`).  NVTX v3 is header-only: with no
// profiler attached a range costs a load and a branch.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace attn {

class TraceRange {
 public:
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

}  // namespace attn
