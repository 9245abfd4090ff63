// common.cuh -- pieces shared by the forward and backward kernels: the device
// error word and the bounded mbarrier wait.
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace fa {

// Device error word of this library (one per device).  A kernel whose bounded
// wait runs out ORs a code into it; the host reads and clears it in
// fa_check_device_error.
__device__ unsigned int g_error_word;

// Codes ORed into the error word: which kernel and which role gave up.
enum : unsigned int {
  kErrFwd = 1u << 0,
  kErrBwdMain = 1u << 1,
  kErrBwdPre = 1u << 2,
  kErrBwdDq = 1u << 3,
  kErrRoleLoad = 1u << 8,
  kErrRoleMma = 1u << 9,
  kErrRoleSoftmax = 1u << 10,
  kErrRoleEpilogue = 1u << 11,
  kErrRoleDrain = 1u << 12,
  kErrRoleDq = 1u << 13,
  kErrAlign = 1u << 14,      // dynamic shared memory base not 1 KiB aligned
  kErrSelfTest = 1u << 15,   // the watchdog self-test kernel gave up (as it must)
  kErrDebugCheck = 1u << 17, // a bounds check of the FA_DEBUG build failed (see dbg_check)
};

// ---------------------------------------------------------- debug build
// Built with -DFA_DEBUG, the kernels check every TMA coordinate, shared-memory
// destination, TMEM column range and directly indexed global address before
// using it.  A failed check records kErrDebugCheck and the role's code in the
// error word, raises the CTA's abort flag and skips the access, so the CTA
// leaves through the same path as a timed-out wait (no trap, no assert).
#ifdef FA_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

__device__ __forceinline__ bool dbg_check(bool cond, unsigned int code, volatile int* abort_flag) {
  if (!kDebugChecks || cond) return true;
  atomicOr(&g_error_word, kErrDebugCheck | code);
  *abort_flag = 1;
  return false;
}

// TMEM address = (lane << 16) | column; a 32x32b access of `cols` columns by
// a warp of a 4-warp group must stay inside the `alloc` allocated columns.
__device__ __forceinline__ bool tmem_range_ok(uint32_t addr, uint32_t base, uint32_t cols,
                                              uint32_t alloc) {
  const uint32_t col = (addr & 0xffffu) - (base & 0xffffu);
  const uint32_t lane = (addr >> 16) - (base >> 16);
  return (addr & 0xffffu) >= (base & 0xffffu) && col + cols <= alloc && lane < 128u &&
         (lane & 31u) == 0u;
}

// Second bound on every wait, in case the global timer were ever to stand
// still: far above any legitimate wait of these kernels.
constexpr uint64_t kMaxWaitIters = 1ull << 28;

// Bounded wait on an mbarrier phase.  Returns true when the phase with the
// given parity has completed; returns false (after recording `code` in the
// error word and raising the CTA's abort flag) once `limit_ns` nanoseconds
// pass, or as soon as another role of the CTA has raised the abort flag.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                             volatile int* abort_flag, unsigned int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint64_t iter = 0;; ++iter) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns || iter > kMaxWaitIters) {
      atomicOr(&g_error_word, code);
      *abort_flag = 1;
      return false;
    }
  }
}

// Bounded wait taken by a whole warp whose lanes then issue warp-collective
// tcgen05.ld / tcgen05.st: all lanes get the same answer (if any lane gave up,
// every lane reports failure), so those instructions are never executed by
// part of a warp.
__device__ __forceinline__ bool wait_bounded_warp(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns, volatile int* abort_flag,
                                                  unsigned int code) {
  const bool ok = wait_bounded(bar, parity, limit_ns, abort_flag, code);
  return __all_sync(0xffffffffu, ok);
}

// Wait that ignores the abort flag: used only to let copies already in flight
// land before the CTA releases its shared memory.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  for (uint64_t iter = 0; !mbar_try_wait(bar, parity); ++iter) {
    if (global_timer_ns() - t0 > limit_ns || iter > kMaxWaitIters) {
      atomicOr(&g_error_word, kErrRoleDrain);
      return;
    }
  }
}

// ------------------------------------------------------ work distribution
// Persistent kernels launch about one CTA per SM; each CTA takes its first
// work item from blockIdx.x and every further one from a per-launch counter
// (one atomicAdd each), so items (ordered longest first) go to whichever CTA
// frees up first.  The counters live here: a launch uses slot (per-device
// launch sequence number mod kSchedSlots), finds it at zero, and the last of
// its CTAs to finish sets it back to zero -- also after a timed-out wait,
// since every CTA leaves through the same exit -- so a replay of the same
// launch (a captured CUDA graph) starts from zero too.  Two launches share a
// slot only kSchedSlots launches apart.
constexpr int kSchedSlots = 1 << 14;
__device__ unsigned int g_sched_next[kSchedSlots];
__device__ unsigned int g_sched_done[kSchedSlots];

// Called once per CTA by one thread after all of the CTA's work: the last CTA
// of the launch clears the slot for the next launch that uses it.
__device__ __forceinline__ void sched_finish(uint32_t slot) {
  __threadfence();
  const unsigned int done = atomicAdd(&g_sched_done[slot], 1u);
  if (done == gridDim.x - 1) {
    atomicExch(&g_sched_next[slot], 0u);
    atomicExch(&g_sched_done[slot], 0u);
  }
}

// Self-test of the bounded wait: one warp waits on an mbarrier that no thread
// ever arrives on.  The wait must give up after limit_ns, record
// kErrSelfTest in the error word, and let the kernel return normally.
__global__ void __launch_bounds__(32, 1) watchdog_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t never_arrived;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&never_arrived), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  __syncthreads();
  (void)wait_bounded_warp(smem_u32(&never_arrived), 0, limit_ns, &abort_flag, kErrSelfTest);
}

}  // namespace fa
