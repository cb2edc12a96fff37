// Self-test of the bounded device-side wait (failure detection without a
// fault).  One CTA holds tensor memory, as the pipeline kernels do, and waits
// through the same bounded wait (mbar_wait) on an mbarrier that nothing ever
// arrives at.  The wait must give up once the wait limit has passed, record
// GMLA_ETIMEOUT in the device error flag, and the CTA must free its tensor
// memory and return, leaving the context usable.  The pages have no
// counterpart; this is the test hook of the library's failure detection.
#pragma once

#include "sm100.cuh"

namespace gmla {
namespace selftest {

using namespace sm100;

// elapsed[0] <- how long the wait lasted (ns); elapsed[1] <- 1 if it gave up.
__global__ void __launch_bounds__(64, 1) wait_kernel(unsigned long long* elapsed) {
  __shared__ __align__(8) uint64_t never;      // an mbarrier nothing arrives at
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&never), 1);
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(&tmem_slot), 32); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0 && lane == 0) {
    const uint64_t t0 = globaltimer_ns();
    const bool ok = mbar_wait(smem_u32(&never), 0, &abort_flag);
    elapsed[0] = globaltimer_ns() - t0;
    elapsed[1] = ok ? 0ull : 1ull;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_slot, 32);
  }
}

}  // namespace selftest
}  // namespace gmla
