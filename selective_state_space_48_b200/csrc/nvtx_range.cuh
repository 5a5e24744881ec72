// nvtx_range.cuh -- NVTX ranges around the library's entry points, so a
// profiler's timeline shows which call enqueued which kernels.  NVTX v3 is
// header-only: without a tool attached each push/pop is a call through a
// function pointer that does nothing, so the ranges cost nothing measurable
// when no profiler is running.  Building with -DMSS_NO_NVTX removes them.
#pragma once

#ifndef MSS_NO_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

namespace sss48 {

class NvtxRange {
 public:
  explicit NvtxRange(const char *name) {
#ifndef MSS_NO_NVTX
    nvtxRangePushA(name);
#else
    (void)name;
#endif
  }
  ~NvtxRange() {
#ifndef MSS_NO_NVTX
    nvtxRangePop();
#endif
  }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

}  // namespace sss48
