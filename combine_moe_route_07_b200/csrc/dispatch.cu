// dispatch.cu -- step 4: permute/scatter token rows into the layout.
//
// "GPU MoE all-to-all" (aicassindra), section "Bucketing: cut the message
// count, not the byte count": the permutation is fused into the kernel that
// stages the rows, so each token row is read once and written k times; and
// section "Latency-bound at decode, bandwidth-bound at prefill": the optional
// lower-precision (e4m3) copy, since the rows feed a matmul that would cast
// them anyway.
//
// Token-major and HBM-bound: no step is a contraction, so the kernel is a
// streaming copy.  A token row is split over G threads; each thread holds
// CPT 16-byte chunks (chunks g, g+G, ... so a warp touches contiguous
// 512-byte runs), loads them once with L1-bypassing loads and issues k
// 16-byte stores per chunk.  Grid: a whole number of waves of resident CTAs.
//
// FP8 variant: the 16 chunks of a 128-channel block sit in 16 aligned lanes;
// amax is a 4-step xor shuffle, then scale = amax/448, inv = 448/amax (IEEE
// division), codes = cvt.rn.satfinite.e4m3x2(x * inv) and 8-byte stores.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 256;

template <int CPT>
__global__ void __launch_bounds__(kThreads)
    dispatch_bf16_kernel(const char* __restrict__ x, const int32_t* __restrict__ dst_pos, int T,
                         int H, int k, int64_t N, char* __restrict__ out, WsHeader* hdr) {
  const int C8 = H >> 3;  // 16-byte chunks per row
  const int G = (C8 + CPT - 1) / CPT;
  const int64_t units = (int64_t)T * G;
  const size_t row_bytes = (size_t)H * 2;
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * kThreads) {
    const int t = (int)(u / G);
    const int g = (int)(u - (int64_t)t * G);
    const char* src = x + (size_t)t * row_bytes;
    uint4 v[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = g + i * G;
      if (c < C8) v[i] = ld16_stream(src + (size_t)c * 16);
    }
    const int32_t* dp = dst_pos + (size_t)t * k;
    for (int j = 0; j < k; ++j) {
      const int p = __ldg(dp + j);
      if (p < 0) continue;
      if (p >= N) {
        if (g == 0) report(hdr, MOE_ERR_DEVICE_RANGE, p);
        continue;
      }
      char* dst = out + (size_t)p * row_bytes;
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = g + i * G;
        if (c < C8) st16(dst + (size_t)c * 16, v[i]);
      }
    }
  }
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

// G is a multiple of 16 so that the 16 threads of a 128-channel block are 16
// aligned lanes of one warp.  The loop runs per warp (all lanes iterate
// together) because the amax reduction shuffles across the block's lanes.
template <int CPT>
__global__ void __launch_bounds__(kThreads)
    dispatch_fp8_kernel(const char* __restrict__ x, const int32_t* __restrict__ dst_pos, int T,
                        int H, int k, int64_t N, uint8_t* __restrict__ out,
                        float* __restrict__ scales, WsHeader* hdr) {
  const int C8 = H >> 3;
  const int G = (((C8 + CPT - 1) / CPT) + 15) & ~15;
  const int nb = H >> 7;  // scale blocks per row
  const int64_t units = (int64_t)T * G;
  const int lane = threadIdx.x & 31;
  const size_t row_bytes = (size_t)H * 2;
  const int64_t warp0 = ((int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31));
  for (int64_t ub = warp0; ub < units; ub += (int64_t)gridDim.x * kThreads) {
    const int64_t u = ub + lane;
    const bool live = u < units;
    const int t = live ? (int)(u / G) : 0;
    const int g = live ? (int)(u - (int64_t)t * G) : 0;
    const char* src = x + (size_t)t * row_bytes;
    uint32_t q[CPT][2];
    float s[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = g + i * G;
      const bool in = live && c < C8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (in) v = ld16_stream(src + (size_t)c * 16);
      float f[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                    bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
      if (amax > 0.0f) {
        const float inv = __fdiv_rn(448.0f, amax);
        s[i] = __fdiv_rn(amax, 448.0f);
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(f[e], inv);
        q[i][0] = pack_e4m3x4(f[0], f[1], f[2], f[3]);
        q[i][1] = pack_e4m3x4(f[4], f[5], f[6], f[7]);
      } else {
        s[i] = 0.0f;
        q[i][0] = 0u;
        q[i][1] = 0u;
      }
    }
    if (!live) continue;
    const int32_t* dp = dst_pos + (size_t)t * k;
    for (int j = 0; j < k; ++j) {
      const int p = __ldg(dp + j);
      if (p < 0) continue;
      if (p >= N) {
        if (g == 0) report(hdr, MOE_ERR_DEVICE_RANGE, p);
        continue;
      }
      uint8_t* dst = out + (size_t)p * H;
      float* sdst = scales + (size_t)p * nb;
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = g + i * G;
        if (c < C8) {
          *reinterpret_cast<uint2*>(dst + (size_t)c * 8) = make_uint2(q[i][0], q[i][1]);
          if ((c & 15) == 0) sdst[c >> 4] = s[i];
        }
      }
    }
  }
}

template <typename K>
int grid_for(K kernel, const LaunchEnv& env, int64_t units) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t need = (units + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)env.num_sms * per_sm;
  int64_t g = need < cap ? need : cap;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_dispatch_bf16(const LaunchEnv& env, const void* x, const int32_t* dst_pos,
                                 int T, int H, int k, int64_t N, void* out, WsHeader* hdr) {
  if (T == 0) return cudaSuccess;
  const int C8 = H / 8;
  const char* xs = static_cast<const char*>(x);
  char* o = static_cast<char*>(out);
  if (C8 >= 512) {
    auto kern = dispatch_bf16_kernel<2>;
    const int grid = grid_for(kern, env, (int64_t)T * ((C8 + 1) / 2));
    kern<<<grid, kThreads, 0, env.stream>>>(xs, dst_pos, T, H, k, N, o, hdr);
  } else {
    auto kern = dispatch_bf16_kernel<1>;
    const int grid = grid_for(kern, env, (int64_t)T * C8);
    kern<<<grid, kThreads, 0, env.stream>>>(xs, dst_pos, T, H, k, N, o, hdr);
  }
  return cudaGetLastError();
}

cudaError_t launch_dispatch_fp8(const LaunchEnv& env, const void* x, const int32_t* dst_pos,
                                int T, int H, int k, int64_t N, void* out, float* scales,
                                WsHeader* hdr) {
  if (T == 0) return cudaSuccess;
  const int C8 = H / 8;
  auto kern = dispatch_fp8_kernel<1>;
  const int G = (C8 + 15) & ~15;
  const int grid = grid_for(kern, env, (int64_t)T * G);
  kern<<<grid, kThreads, 0, env.stream>>>(static_cast<const char*>(x), dst_pos, T, H, k, N,
                                          static_cast<uint8_t*>(out), scales, hdr);
  return cudaGetLastError();
}

}  // namespace moe
