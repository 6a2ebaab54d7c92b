// NVTX ranges over the library's C entry points, so that a timeline profiler
// (Nsight Systems, or any NVTX consumer) shows each call and the kernels and
// copies it issued.  NVTX is header-only: without a tool attached a push or
// pop is a call that returns at once.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace gdn {

struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange &) = delete;
    TraceRange &operator=(const TraceRange &) = delete;
};

}  // namespace gdn

#define GDN_TRACE(name) ::gdn::TraceRange gdn_trace_range_(name)
