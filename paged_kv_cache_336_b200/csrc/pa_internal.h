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
