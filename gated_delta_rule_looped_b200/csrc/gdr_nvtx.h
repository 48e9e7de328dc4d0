// gdr_nvtx.h -- NVTX ranges for the host side of the library: every ABI call and every loop
// launch shows up by name on a profiler's timeline.  NVTX v3 is header-only; with no tool
// attached a range costs a few nanoseconds.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace lt2 {

// A range for the lifetime of a scope.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace lt2
