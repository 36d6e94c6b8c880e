// wait_check.cuh -- a diagnostic kernel for the bounded waits of the decode pipelines.
// Every wait of a decode kernel (a stage barrier, a slot release, the V-gather warp's
// count) gives up after a time limit, sets PA_DEV_TIMEOUT and lets the kernel leave, so
// a pipeline that cannot finish reports an error instead of hanging the GPU.  This kernel
// runs the same two wait helpers against a barrier that nothing arrives on and a count
// that nothing raises, with a caller-chosen limit, so the give-up path can be checked
// without a broken pipeline.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace pkv {

// result[0] / [1]: 1 when the barrier / count wait gave up; result[2] / [3]: how long
// each took, in microseconds (saturated).  One warp; lane 0 waits.
__global__ void pa_wait_check_kernel(int32_t* result, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag, count;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    count = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x != 0) return;
  volatile int* ab = &abort_flag;
  const uint64_t t0 = globaltimer_ns();
  const bool got_bar = mbar_wait_bounded(&bar, 0u, ab, limit_ns);
  const uint64_t t1 = globaltimer_ns();
  const bool got_count = wait_count_bounded(&count, 1, ab, limit_ns);
  const uint64_t t2 = globaltimer_ns();
  const uint64_t cap = 0x7fffffffull;
  result[0] = got_bar ? 0 : 1;
  result[1] = got_count ? 0 : 1;
  result[2] = (int32_t)((t1 - t0) / 1000 < cap ? (t1 - t0) / 1000 : cap);
  result[3] = (int32_t)((t2 - t1) / 1000 < cap ? (t2 - t1) / 1000 : cap);
}

}  // namespace pkv
