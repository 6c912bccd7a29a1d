// trace.h -- an NVTX range named after each C-ABI entry point for the duration of the
// host call, so that what the call enqueues shows up under its name in Nsight Systems.
// NVTX v3 is header-only: without an attached tool each range costs a no-op call.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace spkv {

struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

}  // namespace spkv

#define SPKV_TRACE(name) ::spkv::TraceRange spkv_trace_range_(name)
