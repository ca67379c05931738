// Bounds checks of the debug build.
//
// Built with -DKVPOP_DEBUG (future_attention_targets_b200/build.py, debug
// flavour: libkvpop_debug.so), every kernel checks the index of each
// data-dependent global or shared-memory access before making it.  A failed
// check records, once per word, a code in the debug word the caller
// registered with kvpop_debug_set_word and the access is skipped; nothing
// traps, so the context stays usable and the host reads the code.  In the
// ordinary build KVPOP_IN(...) is the constant `true`: its arguments are not
// evaluated and the checks cost nothing.
//
// Code: KVPOP_ERR_BOUNDS (5) | check site << 8 | kernel << 16.
#pragma once

#include <stdint.h>

namespace kvpop {

enum DebugKernel : int32_t {
  DBG_ROW_LSE = 1,
  DBG_TARGET = 2,
  DBG_KEEP = 3,
  DBG_THRESHOLDS = 4,
  DBG_COMPACT = 5,
  DBG_DECODE = 6,
  DBG_COMBINE = 7,
  DBG_NORM_ROWS = 8,
  DBG_MERGE = 9,
  DBG_SELFTEST = 10,
};

constexpr int32_t kBoundsCode = 5;   // KVPOP_ERR_BOUNDS

__device__ __forceinline__ bool debug_fail(int32_t* word, int32_t kernel, int32_t site) {
  if (word != nullptr) atomicCAS(word, 0, kBoundsCode | (site << 8) | (kernel << 16));
  return false;
}

}  // namespace kvpop

// KVPOP_IN guards an access (false: skip it); KVPOP_CHECK only records
// (for accesses the hardware clips by itself, such as tiled TMA loads).
#ifdef KVPOP_DEBUG
#define KVPOP_IN(cond, word, kernel, site) ((cond) ? true : ::kvpop::debug_fail((word), (kernel), (site)))
#define KVPOP_CHECK(cond, word, kernel, site) ((void)KVPOP_IN(cond, word, kernel, site))
#else
#define KVPOP_IN(cond, word, kernel, site) true
#define KVPOP_CHECK(cond, word, kernel, site) ((void)0)
#endif
