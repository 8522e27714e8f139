// NVTX ranges around the C-ABI entry points, so a timeline profiler shows each
// library call by name. Header-only NVTX v3: with no tool attached a range costs
// a few nanoseconds and nothing is linked.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace tps {

struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

}  // namespace tps

#define TPS_TRACE(name) ::tps::TraceRange tps_trace_range_(name)
