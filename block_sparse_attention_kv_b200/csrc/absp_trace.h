// NVTX ranges around the library's entry points.  Each call that does GPU
// work shows up under its own name on a profiler's timeline, and ncu can
// filter kernels by it (--nvtx --nvtx-include "absp_decode_step_ex/").
// NVTX3 is header-only; with no profiler attached a push or pop costs one
// indirect call to an empty function.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace absp {

struct TraceRange {
    explicit TraceRange(const char* name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange&) = delete;
    TraceRange& operator=(const TraceRange&) = delete;
};

}  // namespace absp

#define ABSP_TRACE(name) const ::absp::TraceRange absp_trace_range_(name)
