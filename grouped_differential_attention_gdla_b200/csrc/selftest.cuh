// selftest.cuh - device-side check of the bounded pipeline wait.
//
// Every wait in the GDLA kernels is an mbarrier poll with a time limit; when
// the limit passes, the kernel records GDLA_ERR_TIMEOUT and unwinds instead
// of hanging.  This kernel runs that same wait on a barrier that nothing ever
// completes, so the failure path can be exercised on a GPU without a fault.
#pragma once

#include "sm100.cuh"

namespace gdla {

__global__ void __launch_bounds__(32, 1) gdla_wait_timeout_kernel(int *status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);  // expects one arrival that never comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  bool ok = mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && threadIdx.x == 0) atomicExch(status, -5 /* GDLA_ERR_TIMEOUT */);
}

}  // namespace gdla
