// last_error.h - the per-thread error text behind pa_last_error(), shared by
// every translation unit of the library.
#pragma once

#include "pagedkv.h"

namespace pagedkv {

// Record a formatted message for pa_last_error() and return `status`.
pa_status fail(pa_status status, const char *fmt, ...)
#if defined(__GNUC__)
    __attribute__((format(printf, 2, 3)))
#endif
    ;

// Clear the message and return PA_OK.
pa_status ok();

} // namespace pagedkv
