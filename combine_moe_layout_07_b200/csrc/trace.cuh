// trace.cuh -- NVTX ranges around the C ABI's entry points: host-side markers that put each call
// on a profiler's timeline next to the kernels it launches (issue and, for the calls that wait,
// the wait itself).  Without a tool attached a range costs a few tens of nanoseconds.
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
