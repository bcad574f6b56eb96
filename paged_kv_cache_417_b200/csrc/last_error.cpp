// last_error.cpp - per-thread text of the last failed call.
#include "last_error.h"

#include <cstdarg>
#include <cstdio>

namespace pagedkv {

namespace {
thread_local char g_last_error[512] = "";
}

pa_status fail(pa_status status, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return status;
}

pa_status ok()
{
    g_last_error[0] = '\0';
    return PA_OK;
}

} // namespace pagedkv

namespace pagedkv {
const char *last_error_text() { return g_last_error; }
} // namespace pagedkv

extern "C" const char *pa_last_error(void) { return pagedkv::last_error_text(); }
