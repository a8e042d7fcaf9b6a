// In-kernel bounds checks of the debug build.
//
// Compiled with ATTN_DEBUG_BOUNDS=1 (libattn_b200_debug.so), ATTN_IN_BOUNDS
// checks an index condition before the access it guards: when the condition
// fails, the access is skipped, ATTN_FAULT_BOUNDS is ORed into the caller's
// error word and the first failing site (attn_bounds_site_t) goes into bits
// 16..23 of it. Nothing traps. A planted site (attn_debug_plant_bounds) is
// reported as failed while the access goes ahead with its real index, so the
// recording path can be exercised without any out-of-range access.
//
// In the release build ATTN_IN_BOUNDS is the constant true and the checks
// compile to nothing.
#pragma once

#include <stdint.h>

#include "attn.h"

#ifndef ATTN_DEBUG_BOUNDS
#define ATTN_DEBUG_BOUNDS 0
#endif

namespace attn {

// ORs ATTN_FAULT_BOUNDS into *flags and sets the site bits if no site is
// recorded yet. The word only ever gains bits, so the compare-and-swap loop
// ends; it is bounded all the same.
__device__ __forceinline__ void bounds_record(int32_t* flags, int site) {
  if (!flags) return;
  int cur = atomicOr(flags, ATTN_FAULT_BOUNDS) | ATTN_FAULT_BOUNDS;
  for (int it = 0; it < 64 && ATTN_FAULT_SITE(cur) == 0; ++it) {
    const int prev = atomicCAS(flags, cur, cur | ((site & 0xff) << 16));
    if (prev == cur) break;
    cur = prev;
  }
}

__device__ __forceinline__ bool bounds_check(bool ok, int site, int32_t* flags, int planted) {
  if (!ok || planted == site) bounds_record(flags, site);
  return ok;
}

}  // namespace attn

#if ATTN_DEBUG_BOUNDS
#define ATTN_IN_BOUNDS(cond, site, flags, planted) ::attn::bounds_check((cond), (site), (flags), (planted))
#else
#define ATTN_IN_BOUNDS(cond, site, flags, planted) true
#endif
