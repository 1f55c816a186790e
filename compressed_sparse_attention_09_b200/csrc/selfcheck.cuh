// Self-check of the library's failure detection: a wait that runs out must
// end, return false to its caller and record kStatusTimeout in the status
// word, and leave the context usable.  One CTA of two warps: warp 0 waits on
// an mbarrier that nothing ever arrives on; warp 1 arrives on a second one
// and waits on it (a wait that completes).  Nothing faults or hangs: the
// first wait ends at the wait limit (csa_set_wait_limit_ns).
#pragma once
#include "sm100.cuh"

namespace csa {

// out[0]: 1 if warp 0's wait reported completion (it must not), out[1]: ns
// warp 0 spent in the wait, out[2]: 1 if warp 1's wait completed.
__global__ void __launch_bounds__(64) wait_selfcheck_kernel(unsigned long long* out) {
  using namespace sm100;
  __shared__ uint64_t bars[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    const uint64_t t0 = global_ns();
    const bool ok = warp_wait(&bars[0], 0);   // no arrival is ever made on bars[0]
    const uint64_t t1 = global_ns();
    if (lane == 0) {
      out[0] = ok ? 1ull : 0ull;
      out[1] = t1 - t0;
    }
  } else {
    if (lane == 0) mbar_arrive(&bars[1]);
    const bool ok = warp_wait(&bars[1], 0);
    if (lane == 0) out[2] = ok ? 1ull : 0ull;
  }
}

}  // namespace csa
