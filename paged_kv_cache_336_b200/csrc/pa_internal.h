// Internal helpers shared by the C-ABI translation units of libpagedkv.
#pragma once

#include <cstdarg>
#include <cstdio>
#include <string>

#include "pagedkv.h"

namespace pagedkv {

// Records a formatted message as the calling thread's last error and returns
// `status` unchanged, so call sites read `return fail(PA_ERR_..., "...")`.
pa_status_t fail(pa_status_t status, const char* fmt, ...);
// Clears the calling thread's last error; returns PA_OK.
pa_status_t ok();

}  // namespace pagedkv

// NVTX ranges around the C-ABI calls that enqueue GPU work, so that a
// timeline (Nsight Systems, or any NVTX consumer) shows each call beside its
// kernels. Compiled in only when the library is built with PAGEDKV_NVTX
// defined (python -m paged_kv_cache_336_b200.build --nvtx); otherwise the
// macro expands to nothing. NVTX v3 is header-only: with no tool attached a
// range costs a test of a function pointer.
#ifdef PAGEDKV_NVTX
#include <nvtx3/nvToolsExt.h>
namespace pagedkv {
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace pagedkv
#define PA_NVTX_RANGE(name) ::pagedkv::NvtxRange pa_nvtx_range_(name)
#else
#define PA_NVTX_RANGE(name) ((void)0)
#endif
