// selftest.cu -- a kernel whose bounded wait runs out: it exercises the
// timeout path of the pipeline waits (mbar_wait: give up after the limit,
// record kDevErrTimeout, return) on a GPU without faulting or hanging it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lt_fault.h"
#include "lt_ptx.cuh"

namespace lt {
namespace {

__global__ void __launch_bounds__(32) lt_selftest_wait_kernel(int* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int s_abort;
  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    // phase 0 never completes: nothing arrives
    mbar_wait(&bar, 0, &s_abort, err, limit_ns);
  }
}

}  // namespace

cudaError_t launch_selftest_wait(int* err, uint64_t limit_ns, cudaStream_t stream) {
  lt_selftest_wait_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace lt
