// selftest.cuh -- exercises the bounded mbarrier wait of the kernels.
//
// One thread waits, through the same mbar_wait the attention kernel uses, on an
// mbarrier that nothing ever arrives on.  The wait gives up after limit_ns,
// raises the device status word and the kernel returns: the path a broken
// pipeline takes, provoked without any fault.
#pragma once

#include "lt_device.cuh"

namespace lt {

__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(unsigned* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, status, limit_ns};
    mbar_wait(&bar, 0, ctl);   // phase 0 never completes
  }
  __syncwarp();
}

}  // namespace lt
