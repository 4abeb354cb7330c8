// Test probe (built by tests/test_gpu_bounded_wait.py, not part of the
// library): a wait on an mbarrier that nothing ever arrives at must give up
// after its time limit and report it, leaving the context usable.
#include <cuda_runtime.h>

#include "gqla.h"
#include "ptx.cuh"

__global__ void wait_for_nothing(int* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    gqla::ptx::mbar_init(&bar, 1);
    gqla::ptx::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = gqla::ptx::mbar_wait_for(&bar, 0, limit_ns);
  if (threadIdx.x == 0) *status = ok ? 0 : GQLA_DEV_TIMEOUT;
}

extern "C" int probe_wait_for_nothing(int* status_dev, unsigned long long limit_ns) {
  wait_for_nothing<<<1, 32>>>(status_dev, limit_ns);
  return (int)cudaGetLastError();
}
