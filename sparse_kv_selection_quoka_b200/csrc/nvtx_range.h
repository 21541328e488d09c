// Host-side NVTX ranges around the library's public calls. Each entry point
// opens a range named after itself for the time it takes to validate and
// enqueue its work, so that a timeline (Nsight Systems) shows the calls and
// the kernels they launched, and a kernel profiler can select one call's
// kernels (ncu --nvtx --nvtx-include "quoka_prefill_chunk/"). With no tool
// attached a range costs a predictable branch.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace quoka {

class NvtxRange {
 public:
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace quoka
