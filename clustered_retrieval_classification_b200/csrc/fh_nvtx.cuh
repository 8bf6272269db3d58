// fh_nvtx.cuh — an NVTX range around each C-ABI entry point, so that a profiler's timeline shows
// which library call issued which kernels.  NVTX v3 is header-only: without an attached tool every
// push and pop is a call through a no-op function pointer.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace fh {

struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace fh

#define FH_NVTX_RANGE(name) const fh::NvtxRange fh_nvtx_range_(name)
