// Optional NVTX ranges around each kernel launch of a call (prologue,
// selection, pair union, attention, sum of squares, RoPE table), so that a
// timeline from Nsight Systems or an `ncu --nvtx` filter shows which part of
// the call a kernel belongs to. Compiled in only with -DLCSA_NVTX (build with
// `python -m block_sparse_video_lcsa_b200.build --nvtx`); otherwise the macro
// is empty and the library does not reference NVTX at all. NVTX v3 is
// header-only: without a profiler attached each range costs a null check.
#pragma once

#ifdef LCSA_NVTX
#include <nvtx3/nvToolsExt.h>

namespace lcsa {
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace lcsa

// one range per scope: the range ends with the enclosing block
#define LCSA_RANGE(name) ::lcsa::NvtxRange lcsa_nvtx_range_(name)
#else
#define LCSA_RANGE(name) \
  do {                   \
  } while (0)
#endif
