// Failure-detection self test: the bounded mbarrier wait of the tensor-core
// pipelines, run against a barrier that nothing will complete.  It must give
// up after its limit and record HS_ERR_TIMEOUT without trapping.

#include "hs_device.cuh"
#include "hs_internal.h"
#include "tc_common.cuh"

namespace hs {
namespace {

__global__ void selftest_wait_kernel(long long limit_ns, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  tc::mbar_init(&bar, 1);  // expects one arrival that never comes
  tc::fence_barrier_init();
  if (!tc::mbar_wait(&bar, 0, limit_ns)) record_status(status, HS_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_selftest_wait(long long limit_ns, int* status, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace hs
