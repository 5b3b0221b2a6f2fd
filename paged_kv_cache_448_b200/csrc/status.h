// status.h — thread-local error message behind pa_last_error().
#pragma once

#include "paged.h"

namespace paged {
// Record a message (printf-style) for pa_last_error() and return `code`.
pa_status fail(pa_status code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
// Forget the previous message (every public call starts with this).
void clear_error();
}  // namespace paged
