// Bounded mbarrier waits and register fences shared by the tcgen05 kernels.
//
// Every wait on an mbarrier phase is bounded: after `limit` cycles of clock64
// (about a second by default) it records WF_ERR_TIMEOUT in the pool's status
// word, raises the CTA's abort flag (which every other waiting role polls) and
// returns false, so a kernel can drain its in-flight copies and MMAs, free TMEM
// and exit instead of spinning forever.
//
// Draining waits for work this CTA has itself issued (TMA copies, MMAs), which
// the hardware completes whatever the other roles do; their bound is a fixed,
// longer one that a shortened per-launch limit does not touch. If even a drain
// runs out, the kernel records WF_ERR_TIMEOUT and still releases its TMEM, so
// no later CTA on the SM blocks on the allocator; the launch's outputs are then
// invalid, which the status word reports.
#pragma once

#include <cstdint>

#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {

constexpr long long kWaitLimit = 2000000000LL;   // ~1 s at 2 GHz (default per-launch limit)
constexpr long long kDrainLimit = 4000000000LL;  // ~2 s: bound of the drain waits

struct Ctx {
  uint64_t *bars;
  volatile int *abort;
  int32_t *status;
  long long limit = kWaitLimit;   // cycles before a wait gives up
};

// Bounded wait on an mbarrier phase. Returns false (and flags the CTA) on
// timeout or when another role has already aborted.
__device__ __forceinline__ bool wait_bar(const Ctx &c, int b, uint32_t parity) {
  uint64_t *bar = c.bars + b;
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    if ((it & 127u) == 0) {
      if (*c.abort) return false;
      if (clock64() - t0 > c.limit) {
        *c.abort = 1;
        record_status(c.status, WF_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait on a phase completed (in part) by the other CTA of a pair:
// acquire at cluster scope.
__device__ __forceinline__ bool wait_bar_cluster(const Ctx &c, int b, uint32_t parity) {
  uint64_t *bar = c.bars + b;
  if (sm100::mbar_try_wait_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (sm100::mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 127u) == 0) {
      if (*c.abort) return false;
      if (clock64() - t0 > c.limit) {
        *c.abort = 1;
        record_status(c.status, WF_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Time-bounded wait used while draining (ignores the abort flag and the
// per-launch limit). Returns false if the drain itself ran out.
__device__ __forceinline__ bool drain_wait(const Ctx &c, int b, uint32_t parity) {
  uint64_t *bar = c.bars + b;
  const long long t0 = clock64();
  while (!sm100::mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kDrainLimit) {
      record_status(c.status, WF_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Keep the compiler from using tcgen05.ld results before tcgen05.wait::ld.
#define WF_REG_FENCE8(r, o)                                                                 \
  asm volatile("" : "+r"(r[o + 0]), "+r"(r[o + 1]), "+r"(r[o + 2]), "+r"(r[o + 3]),         \
               "+r"(r[o + 4]), "+r"(r[o + 5]), "+r"(r[o + 6]), "+r"(r[o + 7]))

__device__ __forceinline__ void reg_fence32(uint32_t *r) {
  WF_REG_FENCE8(r, 0);
  WF_REG_FENCE8(r, 8);
  WF_REG_FENCE8(r, 16);
  WF_REG_FENCE8(r, 24);
}

}  // namespace wf
