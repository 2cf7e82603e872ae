// Internal declarations shared by the library's translation units.
#pragma once
#include <stdint.h>

#include "pkv.h"

// Record a message for pkv_last_error() on this thread and return `s`.
pkv_status pkv_fail(pkv_status s, const char* fmt, ...);

// True when tiles of more than PKV_DECODE_ROWS rows of these shapes run on the
// tcgen05 kernel (16-bit pools of head_dim 64 or 128, fp8 pools of head_dim 128;
// block size >= 8).
bool pkv_tc_capable(int kv_dtype, int head_dim, int block_size);
// CTAs of the tcgen05 kernel resident on the current device, or -1.
int pkv_tc_resident_ctas(int kv_dtype, int head_dim, int block_size);
// True when the decode-sized tiles of these shapes run on the TMA-fed decode kernel (16-bit
// pools with block size >= 8, fp8 pools of head_dim 128 with block size >= 8, NVFP4 pools of
// head_dim 128 with block size >= 16), the one kernel that takes four-head items.
bool pkv_heads4_capable(int kv_dtype, int head_dim, int block_size);

static inline bool pkv_is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }
static inline int pkv_log2(int64_t x) {
  int l = 0;
  while ((int64_t(1) << l) < x) ++l;
  return l;
}
