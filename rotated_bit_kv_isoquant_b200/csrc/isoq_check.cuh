// Index checks of the bounds-checked build (nvcc -DISOQ_CHECK_BOUNDS; build.py --checked).
//
// A kernel guards a computed global, shared or tensor-memory access with
//   if (in_bounds(index_expression_within_extent, status)) { access }
// In the checked build a false condition skips the access and ORs ISOQ_ST_BOUNDS into the
// caller's status word; nothing traps, so a wrong index shows up as a status bit (and a
// parity failure) on the next isoq_get_status.  In the normal build the condition is
// never evaluated and the guard compiles away.
#pragma once

#include <stdint.h>

#include "isoq_common.cuh"

namespace isoq {

#ifdef ISOQ_CHECK_BOUNDS
constexpr bool kCheckBounds = true;
#else
constexpr bool kCheckBounds = false;
#endif

__device__ __forceinline__ bool in_bounds(bool ok, uint32_t* status) {
  if constexpr (kCheckBounds) {
    if (!ok) set_status(status, ISOQ_ST_BOUNDS);
    return ok;
  } else {
    (void)ok;
    (void)status;
    return true;
  }
}

}  // namespace isoq
