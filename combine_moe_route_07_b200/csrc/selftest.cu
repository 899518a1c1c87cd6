// selftest.cu -- a self-test of the device error path of the bounded waits
// (no page has a counterpart; it exists so the failure handling can be
// exercised on a GPU without provoking any fault).  One warp arms an mbarrier
// for 16 bytes that no copy will ever deliver and waits on it with the same
// bounded wait the bulk-copy kernels use.  When the limit runs out it records
// MOE_ERR_DEVICE_TIMEOUT in the workspace header, detail = the microseconds
// it waited, and returns; nothing is in flight, so the context stays usable.
#include <limits.h>

#include "bulk.cuh"
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(WsHeader* hdr, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(&bar, 16u);  // the arrival happens; the 16 bytes never do
  }
  __syncwarp();
  const uint64_t t0 = global_ns();
  const bool ok = mbar_wait_bounded(&bar, 0u, timeout_ns);
  if (!ok && threadIdx.x == 0) {
    const uint64_t us = (global_ns() - t0) / 1000u;
    report(hdr, MOE_ERR_DEVICE_TIMEOUT, us > (uint64_t)INT_MAX ? INT_MAX : (int)us);
  }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(const LaunchEnv& env, WsHeader* hdr,
                                         uint64_t timeout_ns) {
  wait_timeout_kernel<<<1, 32, 0, env.stream>>>(hdr, timeout_ns);
  return cudaGetLastError();
}

}  // namespace moe
