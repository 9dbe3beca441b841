// Internal helpers shared by the library's translation units (not part of the ABI).
#pragma once
#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/pkv.h"

namespace pkv {

// Record a printf-style message as the calling thread's last error and return code.
pkv_status fail(pkv_status code, const char *fmt, ...);
void clear_error();

}  // namespace pkv
