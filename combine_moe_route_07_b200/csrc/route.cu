// route.cu -- step 1: top-k router with a selection-only per-expert bias.
//
// "19. All-to-all" (ai-from-scratch), section "Why the router can ruin your
// day": the per-expert balancing bias enters the top-k decision and nothing
// else; the mix weights come from the router's own scores.
//
// One warp per token.  Lane l holds experts l, l+32, l+64, ... in registers,
// as order-preserving 32-bit codes of key = logit + bias.  Each of the k
// rounds is two warp reductions in hardware (redux.sync): the largest code,
// then the lowest expert id among lanes holding it, which is the tie rule.
// Gates are a softmax of the selected raw logits evaluated in fp64 (k values
// per token, off the memory-bound critical path) and rounded to fp32 once.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// Finite fp32 -> uint32 with the same order; -0 folds onto +0 first so the
// two compare equal.  No non-NaN key maps to 0, which marks "taken".
__device__ __forceinline__ uint32_t order_code(float f) {
  if (f == 0.0f) f = 0.0f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

template <int NK>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits,
                                                    const float* __restrict__ bias, int T, int E,
                                                    int k, int renorm, int32_t* __restrict__ ids,
                                                    float* __restrict__ gates, WsHeader* hdr) {
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;

  float b[NK];
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int e = lane + 32 * i;
    b[i] = (bias != nullptr && e < E) ? __ldg(bias + e) : 0.0f;
  }

  for (int t = warp; t < T; t += nwarps) {
    const float* row = logits + (size_t)t * E;
    float raw[NK];
    uint32_t code[NK];
    bool nan_key = false;
#pragma unroll
    for (int i = 0; i < NK; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        raw[i] = __ldcs(row + e);  // read once: streaming
        const float key = __fadd_rn(raw[i], b[i]);
        nan_key |= (key != key);
        code[i] = order_code(key);
      } else {
        raw[i] = -INFINITY;
        code[i] = 0u;
      }
    }
    if (__any_sync(kFull, nan_key) && lane == 0) report(hdr, MOE_ERR_DEVICE_NAN, t);

    int sel_e = 0;
    float sel_raw = 0.0f;
    for (int j = 0; j < k; ++j) {
      // this lane's best remaining expert (strict >: lowest index on ties)
      uint32_t best = 0u;
      int bi = 0;
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if (code[i] > best) {
          best = code[i];
          bi = i;
        }
      const uint32_t top = __reduce_max_sync(kFull, best);
      const uint32_t cand = (best == top) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu;
      const uint32_t win = __reduce_min_sync(kFull, cand);
      float r = 0.0f;
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if ((uint32_t)(lane + 32 * i) == win) {
          code[i] = 0u;
          r = raw[i];
        }
      r = __shfl_sync(kFull, r, (int)(win & 31u));
      if (lane == j) {
        sel_e = (int)win;
        sel_raw = r;
      }
    }

    float g;
    if (renorm) {
      const float m = warp_max(lane < k ? sel_raw : -INFINITY);
      const double ex = (lane < k) ? exp((double)sel_raw - (double)m) : 0.0;
      const double den = warp_sum(ex);
      g = (float)(ex / den);
    } else {
      float lm = -INFINITY;
#pragma unroll
      for (int i = 0; i < NK; ++i) lm = fmaxf(lm, raw[i]);
      const float m = warp_max(lm);
      double part = 0.0;
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if (lane + 32 * i < E) part += exp((double)raw[i] - (double)m);
      const double den = warp_sum(part);
      g = (float)(exp((double)sel_raw - (double)m) / den);
    }
    if (lane < k) {
      ids[(size_t)t * k + lane] = sel_e;
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
