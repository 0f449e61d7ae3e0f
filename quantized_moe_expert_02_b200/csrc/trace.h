// NVTX ranges around the library's entry points: a profiler that records
// NVTX (Nsight Systems, ncu's --nvtx filters) sees one named range per call
// on the calling host thread.  Header-only NVTX v3: with no tool attached
// a push or pop is one test of an unset function pointer.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace moe {

struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

}  // namespace moe

// One range named after the enclosing entry point, closed on every return.
#define MOE_TRACE() ::moe::TraceRange moe_trace_range_(__func__)
