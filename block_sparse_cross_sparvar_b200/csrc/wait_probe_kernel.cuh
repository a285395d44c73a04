// Self-test of the bounded waits every kernel of the library uses: one thread
// waits on a shared-memory mbarrier that nothing completes, with the same helper
// and the same give-up path as the attention pipeline (abort flag raised,
// timeout bit ORed into the caller's status word), then the kernel returns.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace sparvar {

// result[0]: 1 if the wait saw the phase complete, 0 if it gave up;
// result[1]: the abort flag afterwards; result[2]: microseconds spent waiting.
__global__ void __launch_bounds__(32) wait_probe_kernel(uint64_t limit_ns, int32_t err_bit,
                                                        int32_t* dev_status, int32_t* result) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // phase 0 needs one arrival, which never comes
    abort_sh = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    volatile int* abort_flag = &abort_sh;
    const uint64_t t0 = global_timer_ns();
    const bool done = mbar_wait(&bar, 0u, abort_flag, dev_status, err_bit, limit_ns);
    const uint64_t us = (global_timer_ns() - t0) / 1000u;
    result[0] = done ? 1 : 0;
    result[1] = *abort_flag;
    result[2] = static_cast<int32_t>(us < 0x7fffffffu ? us : 0x7fffffffu);
  }
}

}  // namespace sparvar
