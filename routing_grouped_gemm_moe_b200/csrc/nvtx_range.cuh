// NVTX range around a C-ABI entry point, named after the function: a profiler
// timeline (Nsight Systems) then shows the library's calls around their
// kernels.  NVTX is header-only here and does nothing unless a tool is
// attached.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace moe {

struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace moe

#define MOE_NVTX_RANGE() ::moe::NvtxRange moe_nvtx_range_(__func__)
