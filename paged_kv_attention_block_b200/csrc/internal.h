// Internal declarations shared by the library's translation units.
#pragma once
#include <stdint.h>

#include "pkv.h"

// Record a message for pkv_last_error() on this thread and return `s`.
pkv_status pkv_fail(pkv_status s, const char* fmt, ...);

static inline bool pkv_is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }
static inline int pkv_log2(int64_t x) {
  int l = 0;
  while ((int64_t(1) << l) < x) ++l;
  return l;
}
