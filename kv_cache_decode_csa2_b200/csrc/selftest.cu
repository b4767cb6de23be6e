// Self-test of the bounded waits.  Every wait of the co-resident kernels (the
// grid barrier of select, reindex and attention) and of the TMA and
// tensor-core pipelines (the mbarrier wait) gives up after a time limit,
// records CSA2_ERR_TIMEOUT and lets its kernel return, so a wait that cannot
// end never hangs the device.  This kernel runs one such wait on something
// that never happens, with a caller-chosen short limit, so that a test can
// check the give-up path without a fault or a hang.
#include "csa2_device.cuh"
#include "internal.h"
#include "select_common.cuh"

namespace csa2 {

namespace {

__global__ void __launch_bounds__(64) wait_selftest_kernel(int32_t kind, uint64_t limit_ns, uint32_t* counter,
                                                           int32_t* status) {
  if (kind == 0) {
    sel_grid_sync(counter, 2u, status, limit_ns);   // a barrier of two CTAs, in a grid of one
    return;
  }
  __shared__ uint64_t bar;
  __shared__ int32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival completes a phase; none comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag, limit_ns)) record_error(status, CSA2_ERR_TIMEOUT);
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_selftest(int32_t kind, uint64_t limit_ns, uint32_t* counter, int32_t* status,
                                 cudaStream_t st) {
  wait_selftest_kernel<<<1, 64, 0, st>>>(kind, limit_ns, counter, status);
  return cudaGetLastError();
}

}  // namespace csa2
