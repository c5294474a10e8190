// Per-call tracing: every C-ABI call that queues device work opens a named
// NVTX range for the duration of the host call ("pkv:<call name>"), so that a
// profiler attached to the process (Nsight Systems, or ncu's --nvtx
// filtering) attributes the launches to the library call that made them.
// NVTX is header-only; with no tool attached a range costs one branch.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace pkv {

class TraceRange {
public:
    explicit TraceRange(const char* name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange&) = delete;
    TraceRange& operator=(const TraceRange&) = delete;
};

}  // namespace pkv

#define PKV_TRACE(name) ::pkv::TraceRange pkv_trace_range_("pkv:" name)
