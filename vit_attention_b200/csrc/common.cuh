// Shared device-side pieces: the workspace status word and the bounded
// mbarrier wait every kernel uses (no wait in this library can spin forever).
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"
#include "vggt_attn.h"

namespace vggt {

// Workspace layout: [0, 256) status block, then the packed tensors.
constexpr size_t kStatusBytes = 256;
// status[0]: first error code recorded (0 = none); status[1]: tag of the wait that expired.
struct StatusBlock {
  int code;
  uint32_t where;
};

__device__ __forceinline__ void record_error(int* status, int code, uint32_t where) {
  if (atomicCAS(status, 0, code) == 0) {
    reinterpret_cast<volatile uint32_t*>(status)[1] = where;
  }
}

// Device-side bounds checks of the debug build (compiled with -DVGGT_DEBUG):
// a failed check records VGGT_ATTN_ERR_BOUNDS with the check's tag in the
// status word and the access it guards is skipped instead of faulting.  In
// the release build the checks compile to `true`.
#ifdef VGGT_DEBUG
#define VGGT_DBG_BOUNDS(cond, status, where) \
  ((cond) ? true : (::vggt::record_error((status), VGGT_ATTN_ERR_BOUNDS, (where)), false))
#else
#define VGGT_DBG_BOUNDS(cond, status, where) true
#endif

__device__ __forceinline__ bool status_is_set(const int* status) {
  return *reinterpret_cast<const volatile int*>(status) != 0;
}

// Wait for the phase of `bar` with parity `parity` to complete.
// Gives up (returns false) when `*abort` is raised by another role of the
// CTA, or after `timeout_ns`, in which case it raises `*abort` and records
// VGGT_ATTN_ERR_TIMEOUT with `where` in the status word.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort, int* status,
                                             uint64_t timeout_ns, uint32_t where) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        *abort = 1;
        record_error(status, VGGT_ATTN_ERR_TIMEOUT, where);
        return false;
      }
    }
  }
}

// Teardown variant: ignores the abort flag (used to drain copies / MMAs that
// are already in flight before the CTA releases its memory).
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

}  // namespace vggt
