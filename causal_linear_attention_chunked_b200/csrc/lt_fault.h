// lt_fault.h -- host-side fault injection and the bounded-wait self-test,
// for testing the error paths without a GPU fault.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

namespace lt {

// LT_FAULT_WORKSPACE_ALLOC set (to anything but "0") in the environment
// makes every stream-ordered workspace allocation of the forward pass report
// cudaErrorMemoryAllocation before anything is enqueued.  Off by default.
inline bool injected_workspace_alloc_failure() {
  const char* f = getenv("LT_FAULT_WORKSPACE_ALLOC");
  return f != nullptr && f[0] != '\0' && !(f[0] == '0' && f[1] == '\0');
}

// One warp waits, through the same bounded mbarrier wait every kernel uses,
// on a barrier nothing arrives on; after limit_ns it records a timeout in
// the device error word and returns.
cudaError_t launch_selftest_wait(int* err, uint64_t limit_ns, cudaStream_t stream);

}  // namespace lt
