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
};

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
