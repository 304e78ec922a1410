// NVTX ranges around the library's entry points, so that a profiler timeline (Nsight Systems,
// Nsight Compute's range filters) shows each C ABI call and the kernels it enqueued.  NVTX v3
// is header-only: without a tool attached each push and pop is a check of a function pointer.
#pragma once
#include <nvtx3/nvToolsExt.h>

namespace dpclip {

inline nvtxDomainHandle_t nvtx_domain() {
  static nvtxDomainHandle_t d = nvtxDomainCreateA("dpclip");
  return d;
}

// Pushes a range named after the entry point on construction, pops it on destruction.
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) {
    nvtxEventAttributes_t a = {};
    a.version = NVTX_VERSION;
    a.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
    a.messageType = NVTX_MESSAGE_TYPE_ASCII;
    a.message.ascii = name;
    nvtxDomainRangePushEx(nvtx_domain(), &a);
  }
  ~NvtxRange() { nvtxDomainRangePop(nvtx_domain()); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace dpclip

#define DP_NVTX_RANGE() ::dpclip::NvtxRange dp_nvtx_range_(__func__)
