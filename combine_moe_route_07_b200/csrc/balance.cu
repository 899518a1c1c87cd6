// balance.cu -- the aux-loss-free balancing step: the per-expert bias update
// from the batch's histogram.
//
// "19. All-to-all" (ai-from-scratch), section "Why the router can ruin your
// day": a bias per expert, bumped up or down based on recent load and used
// only for the top-k decision.  Here: b_e += gamma * sign(mean - load_e) with
// mean = T*k/E, the sign taken exactly in integers (T*k - E*load_e), so an
// expert at the mean keeps its bias.  One binary32 addition per expert.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    bias_update_kernel(const int32_t* __restrict__ counts, int E, int64_t assignments,
                       float gamma, float* __restrict__ bias) {
  pdl_wait();  // counts (and the bias) may come from the kernels launched before
  pdl_trigger();
  for (int e = blockIdx.x * kThreads + threadIdx.x; e < E; e += gridDim.x * kThreads) {
    const int64_t d = assignments - (int64_t)E * __ldg(counts + e);
    if (d > 0)
      bias[e] = __fadd_rn(bias[e], gamma);
    else if (d < 0)
      bias[e] = __fsub_rn(bias[e], gamma);
  }
}

}  // namespace

cudaError_t launch_bias_update(const LaunchEnv& env, const int32_t* counts, int E,
                               int64_t assignments, float gamma, float* bias) {
  const int grid = (E + kThreads - 1) / kThreads;
  return launch_pdl(env, bias_update_kernel, dim3(grid > 0 ? grid : 1), dim3(kThreads), 0, counts,
                    E, assignments, gamma, bias);
}

}  // namespace moe
