// status.cpp — thread-local error message behind pa_last_error().
#include "status.h"

#include <cstdarg>
#include <cstdio>

namespace paged {
namespace {
thread_local char g_message[512] = "";
}

pa_status fail(pa_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_message, sizeof(g_message), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_message[0] = '\0'; }

}  // namespace paged

extern "C" PA_API const char* pa_last_error(void) { return paged::g_message; }
