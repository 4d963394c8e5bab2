// nvtx_range.cuh -- an NVTX range around each public entry point, named after the entry
// point, so that a timeline tool shows which library call enqueued which kernels.  NVTX is
// header-only here; without a tool attached (no NVTX_INJECTION64_PATH) the push and pop
// return at once.
#pragma once
#include <nvtx3/nvToolsExt.h>

namespace lsa {
struct AbiRange {
    explicit AbiRange(const char *name) { nvtxRangePushA(name); }
    ~AbiRange() { nvtxRangePop(); }
    AbiRange(const AbiRange &) = delete;
    AbiRange &operator=(const AbiRange &) = delete;
};
}  // namespace lsa

#define LSA_ABI_RANGE() const ::lsa::AbiRange lsa_abi_range_(__func__)
