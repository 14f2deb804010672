// cf_trace.h -- NVTX ranges around the library's entry points, so a
// profiler timeline (nsys, or ncu --nvtx filters) shows which call enqueued
// which kernels.  NVTX v3 is header-only: without an attached tool every
// range is a no-op.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace cf {

struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange &) = delete;
    TraceRange &operator=(const TraceRange &) = delete;
};

}  // namespace cf
