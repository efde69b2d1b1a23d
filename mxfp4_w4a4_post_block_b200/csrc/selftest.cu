// Self-test of the bounded barrier wait every libbatq kernel uses.
//
// k_wait_selftest waits on an mbarrier that nothing ever arrives on, with a
// short limit; the wait gives up, sets the data-timeout bit in the device
// error word and the kernel returns.  This exercises the failure path of the
// kernels (a stage that never lands) without any copy in flight.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/batq.h"
#include "kernels.h"
#include "ptx.cuh"

namespace batq {
namespace {

__global__ void k_wait_selftest(uint64_t limit_ns, unsigned* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    if (!mbar_wait(&bar, 0, limit_ns)) set_error(err, kErrDataTimeout);
  }
}

}  // namespace

cudaError_t launch_wait_selftest(uint64_t limit_ns, unsigned* err, cudaStream_t stream) {
  k_wait_selftest<<<1, 32, 0, stream>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace batq
