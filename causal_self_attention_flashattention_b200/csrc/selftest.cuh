// Self-test of the failure path every kernel of the library shares: a bounded
// mbarrier wait that gives up, records its site in the device status word,
// raises the CTA's abort flag, and lets the CTA's other roles wind down and
// free their tensor memory instead of waiting out their own limits.
//
// One CTA of two warps. Warp 0 holds a tensor-memory allocation and waits
// (lane 0) on an mbarrier that nothing ever arrives on, with the caller's
// short limit. Warp 1 (lane 0) waits on the same barrier with the library's
// 2 s limit, as any kernel role would; it returns once warp 0 raises the abort
// flag, without recording anything. Then warp 0 frees its tensor memory and
// the kernel returns. Nothing traps, faults or spins without a bound: the
// longest any thread can wait is the 2 s limit.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace ga {

// The longest limit the self-test entry point accepts (1 s), below the 2 s
// limit of the waiter that must wind down on the abort flag instead.
constexpr unsigned long long kMaxSelftestLimitNs = 1000000000ull;

namespace selftest {

constexpr int kThreads = 64;
constexpr uint32_t kTmemCols = 32;

__global__ void __launch_bounds__(kThreads, 1) wait_timeout_kernel(uint64_t limit_ns) {
  __shared__ uint64_t never;  // no thread arrives on this barrier
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort = &abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (lane == 0) {
    if (warp == 0)
      mbar_wait_limit(&never, 0, kSiteSelftestWait, abort, limit_ns);
    else
      mbar_wait(&never, 0, kSiteSelftestPeer, abort);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace selftest
}  // namespace ga
