// Device side of the workspace status block: how a kernel whose bounded wait
// ran out records the failure and tells the other CTAs of its launch to stop.
#pragma once

#include "apb_internal.h"

namespace apb {

__device__ __forceinline__ void record_failure(DeviceStatus* st, uint32_t where, uint32_t tile) {
  if (atomicOr(&st->sticky, kErrWaitTimeout) == 0u) {
    st->where = where;
    st->tile = tile;
  }
  atomicExch(&st->abort, 1u);
  __threadfence();
}

}  // namespace apb
