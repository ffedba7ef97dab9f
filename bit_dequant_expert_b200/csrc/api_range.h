// A named NVTX range around each C-ABI call, so that a timeline tool
// (Nsight Systems and the like) shows the calls by name above their
// kernels.  With no tool attached the push and pop return at once.
#ifndef MOE_API_RANGE_H
#define MOE_API_RANGE_H

#include <nvtx3/nvToolsExt.h>

namespace moe {

class ApiRange {
public:
    explicit ApiRange(const char* name) { nvtxRangePushA(name); }
    ~ApiRange() { nvtxRangePop(); }
    ApiRange(const ApiRange&) = delete;
    ApiRange& operator=(const ApiRange&) = delete;
};

}  // namespace moe

#endif
