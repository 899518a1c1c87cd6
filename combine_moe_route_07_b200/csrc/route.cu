// route.cu -- step 1 on its own: one warp per token (see route_core.cuh).
#include "common.cuh"
#include "kernels.h"
#include "route_core.cuh"

namespace moe {

template <int NK>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits,
                                                    const float* __restrict__ bias, int T, int E,
                                                    int k, int renorm, int32_t* __restrict__ ids,
                                                    float* __restrict__ gates, WsHeader* hdr) {
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  float b[NK];
  load_bias<NK>(bias, E, lane, b);
  for (int t = warp; t < T; t += nwarps) {
    int e;
    float g;
    bool nan_key;
    route_token<NK>(logits + (size_t)t * E, b, E, k, renorm, lane, e, g, nan_key);
    if (nan_key && lane == 0) report(hdr, MOE_ERR_DEVICE_NAN, t);
    if (lane < k) {
      ids[(size_t)t * k + lane] = e;
      gates[(size_t)t * k + lane] = g;
    }
  }
}

template <int NK>
static cudaError_t launch_route_nk(const LaunchEnv& env, const float* logits, const float* bias,
                                   int T, int E, int k, int renorm, int32_t* ids, float* gates,
                                   WsHeader* hdr) {
  const int threads = 256;
  const int warps_per_block = threads / 32;
  int blocks = (T + warps_per_block - 1) / warps_per_block;
  const int cap = env.num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  route_kernel<NK><<<blocks, threads, 0, env.stream>>>(logits, bias, T, E, k, renorm, ids, gates,
                                                       hdr);
  return cudaGetLastError();
}

cudaError_t launch_route(const LaunchEnv& env, const float* logits, const float* bias, int T,
                         int E, int k, int renorm, int32_t* ids, float* gates, WsHeader* hdr) {
  const int nk = (E + 31) / 32;
  if (nk <= 1) return launch_route_nk<1>(env, logits, bias, T, E, k, renorm, ids, gates, hdr);
  if (nk <= 2) return launch_route_nk<2>(env, logits, bias, T, E, k, renorm, ids, gates, hdr);
  if (nk <= 4) return launch_route_nk<4>(env, logits, bias, T, E, k, renorm, ids, gates, hdr);
  if (nk <= 8) return launch_route_nk<8>(env, logits, bias, T, E, k, renorm, ids, gates, hdr);
  if (nk <= 16) return launch_route_nk<16>(env, logits, bias, T, E, k, renorm, ids, gates, hdr);
  return launch_route_nk<32>(env, logits, bias, T, E, k, renorm, ids, gates, hdr);
}

}  // namespace moe
