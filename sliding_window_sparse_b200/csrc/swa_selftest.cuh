// swa_selftest.cuh -- a self-contained check of the bounded waits every
// attention kernel relies on for failure detection.
//
// One CTA of 128 threads and two mbarriers, no copies and no tensor memory.
// Warp 0 lane 0 waits on barrier A with a short limit; warps 1-3 wait, every
// lane, on barrier B through mbar_wait_warp with the kernels' usual limit.
//  - arrive == 0: nobody arrives on either barrier.  Lane 0 of warp 0 gives
//    up after limit_ns, records SWA_DEV_TIMEOUT and raises the abort flag;
//    warps 1-3 then give up within a few polls instead of waiting out their
//    own (much longer) limit.
//  - arrive != 0: thread 0 arrives on both barriers before anyone waits, so
//    every wait succeeds and the status word is left alone.
// result[w] (w = 0..3) counts the lanes of warp w whose wait succeeded (warp
// 0 has one waiting lane); result[4] is the CTA's elapsed time in
// microseconds from before the first wait to after the last.
#pragma once
#include <cstdint>

#include "sm100.cuh"

namespace swa {

__global__ void __launch_bounds__(128, 1)
    selftest_wait_kernel(uint64_t limit_ns, int arrive, int32_t *result) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_word;
  __shared__ int ok_count[4];
  __shared__ unsigned long long t_start;
  const uint32_t bar_a = smem_u32(&bars[0]), bar_b = smem_u32(&bars[1]);
  volatile int *abort_flag = &abort_word;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar_a, 1);
    mbar_init(bar_b, 1);
    *abort_flag = 0;
    for (int w = 0; w < 4; ++w) ok_count[w] = 0;
    fence_barrier_init();
    if (arrive) {
      mbar_arrive(bar_a);
      mbar_arrive(bar_b);
    }
    t_start = global_ns();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0 && mbar_wait_limit(bar_a, 0, abort_flag, limit_ns)) atomicAdd(&ok_count[0], 1);
  } else {
    const bool ok = mbar_wait_warp(bar_b, 0, abort_flag);
    if (ok) atomicAdd(&ok_count[warp], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 0; w < 4; ++w) result[w] = ok_count[w];
    result[4] = static_cast<int32_t>((global_ns() - t_start) / 1000ull);
  }
}

}  // namespace swa
