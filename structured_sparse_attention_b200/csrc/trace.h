// trace.h -- NVTX ranges around the library's entry points (host side).
//
// Each C entry point that launches work opens a range named after itself for the
// duration of the call, so the launches of one call group together in a timeline tool
// (Nsight Systems, or ncu's --nvtx filters).  NVTX 3 is header-only: with no tool
// attached a range costs a few nanoseconds and does nothing.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace ssa {

struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange &) = delete;
    TraceRange &operator=(const TraceRange &) = delete;
};

}  // namespace ssa
