// Library-wide C-ABI helpers: version, status names, per-thread last error.
#include <cstdarg>
#include <cstdio>
#include <string>

#include "pa_internal.h"

namespace pagedkv {

thread_local std::string g_last_error;

pa_status_t fail(pa_status_t status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

pa_status_t ok() {
  g_last_error.clear();
  return PA_OK;
}

}  // namespace pagedkv

extern "C" {

const char* pa_version(void) { return "pagedkv 0.1 sm_100a"; }

const char* pa_last_error_string(void) { return pagedkv::g_last_error.c_str(); }

const char* pa_status_string(pa_status_t status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_NO_FREE_BLOCKS: return "PA_ERR_NO_FREE_BLOCKS";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
  }
  return "PA_ERR_UNKNOWN";
}

}  // extern "C"
