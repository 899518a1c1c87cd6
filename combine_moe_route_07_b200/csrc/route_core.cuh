// route_core.cuh -- one token's top-k selection and gates, executed by one
// warp.  Shared by the standalone route kernel and the fused route + layout
// kernel.
//
// "19. All-to-all" (ai-from-scratch), section "Why the router can ruin your
// day": the per-expert balancing bias enters the top-k decision and nothing
// else; the mix weights come from the router's own scores.
//
// Lane l holds experts l, l+32, l+64, ... in registers as order-preserving
// 32-bit codes of key = logit + bias.  Each of the k rounds is two hardware
// warp reductions (redux.sync): the largest code, then the lowest expert id
// among the lanes holding it, which is the tie rule.  The gates are a softmax
// of the selected RAW logits evaluated in fp64 (k values per token, off the
// memory-bound path) and rounded to fp32 once.
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {

// Finite fp32 -> uint32 with the same order; -0 folds onto +0 first so the
// two compare equal.  No non-NaN key maps to 0, which marks "taken".
__device__ __forceinline__ uint32_t order_code(float f) {
  if (f == 0.0f) f = 0.0f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

template <int NK>
__device__ __forceinline__ void load_bias(const float* bias, int E, int lane, float (&b)[NK]) {
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int e = lane + 32 * i;
    b[i] = (bias != nullptr && e < E) ? __ldg(bias + e) : 0.0f;
  }
}

// Route the token whose logits start at `row`.  On return lane j < k holds
// slot j: expert `sel_e` and gate `gate`.  `nan_key` is set on every lane if
// any key of the token was NaN.
template <int NK>
__device__ __forceinline__ void route_token(const float* __restrict__ row, const float (&b)[NK],
                                            int E, int k, int renorm, int lane, int& sel_e,
                                            float& gate, bool& nan_key) {
  float raw[NK];
  uint32_t code[NK];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      raw[i] = __ldcs(row + e);  // read once: streaming
      const float key = __fadd_rn(raw[i], b[i]);
      bad |= (key != key);
      code[i] = order_code(key);
    } else {
      raw[i] = -INFINITY;
      code[i] = 0u;
    }
  }
  nan_key = __any_sync(kFull, bad);

  sel_e = 0;
  float sel_raw = 0.0f;
  for (int j = 0; j < k; ++j) {
    uint32_t best = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < NK; ++i)
      if (code[i] > best) {  // strict: the lowest index wins ties
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

  if (renorm) {
    const float m = warp_max_f(lane < k ? sel_raw : -INFINITY);
    const double ex = (lane < k) ? exp((double)sel_raw - (double)m) : 0.0;
    const double den = warp_sum_d(ex);
    gate = (float)(ex / den);
  } else {
    float lm = -INFINITY;
#pragma unroll
    for (int i = 0; i < NK; ++i) lm = fmaxf(lm, raw[i]);
    const float m = warp_max_f(lm);
    double part = 0.0;
#pragma unroll
    for (int i = 0; i < NK; ++i)
      if (lane + 32 * i < E) part += exp((double)raw[i] - (double)m);
    const double den = warp_sum_d(part);
    gate = (float)(exp((double)sel_raw - (double)m) / den);
  }
}

}  // namespace moe
