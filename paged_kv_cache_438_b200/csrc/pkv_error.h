// Thread-local error message shared by the C-ABI entry points of libpagedkv.
#pragma once

#include <cstdarg>
#include <cstdio>

#include "../../include/pagedkv.h"

namespace pkv {

// Defined once in pkv_allocator.cpp.
char* error_buffer();

inline int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(error_buffer(), 512, fmt, ap);
  va_end(ap);
  return code;
}

inline int ok() {
  error_buffer()[0] = '\0';
  return PKV_OK;
}

}  // namespace pkv
