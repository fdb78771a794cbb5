// Check of the bounded-wait mechanism every pipelined kernel relies on: a
// kernel waits on an mbarrier that nothing arrives on, with the library's
// bounded wait; the wait must give up after the limit and set the timeout bit
// of the device error word, leaving the context usable.  Nothing here faults,
// traps or spins without a limit.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

__global__ void wait_check_kernel(uint64_t limit_ns, int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !ptx::mbar_wait(&bar, 0, nullptr, limit_ns)) flag_error(err, MOE_DEVERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_check(int64_t limit_ns, cudaStream_t s, const Ctx& ctx) {
  wait_check_kernel<<<1, 32, 0, s>>>((uint64_t)limit_ns, ctx.err);
  return cudaGetLastError();
}

}  // namespace moe
