// combine.cu -- step 5: inverse-permutation gather, gate-weighted sum,
// shared-expert and residual add.
//
// "GPU MoE all-to-all" (aicassindra), section "Two collectives per layer, and
// what each one moves": k partial results come back along the inverse
// permutation and are scaled by the router's gate weights.  "MoE All-to-All
// Dispatch and Ragged Routing", section "Returning Tokens to the Original
// GPU": the residual x + dx is formed where x lives.  "19. All-to-all",
// section "Why the router can ruin your day": a dropped slot counts as if the
// token skipped that expert.
//
// Token-major gather, HBM-bound.  A token row is split over G threads of CPT
// 16-byte chunks; each thread issues the loads of up to kBatch slots before
// using any of them (independent 16-byte loads in flight), then accumulates
// in fp32 in slot order j = 0..k-1 with explicit round-to-nearest FMAs, adds
// the shared-expert row and the residual row, and rounds to bf16 once.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 8;

__device__ __forceinline__ void fma8(float (&acc)[8], float g, const uint4& v) {
  acc[0] = __fmaf_rn(g, bf16lo(v.x), acc[0]);
  acc[1] = __fmaf_rn(g, bf16hi(v.x), acc[1]);
  acc[2] = __fmaf_rn(g, bf16lo(v.y), acc[2]);
  acc[3] = __fmaf_rn(g, bf16hi(v.y), acc[3]);
  acc[4] = __fmaf_rn(g, bf16lo(v.z), acc[4]);
  acc[5] = __fmaf_rn(g, bf16hi(v.z), acc[5]);
  acc[6] = __fmaf_rn(g, bf16lo(v.w), acc[6]);
  acc[7] = __fmaf_rn(g, bf16hi(v.w), acc[7]);
}

__device__ __forceinline__ void add8(float (&acc)[8], const uint4& v) {
  acc[0] = __fadd_rn(acc[0], bf16lo(v.x));
  acc[1] = __fadd_rn(acc[1], bf16hi(v.x));
  acc[2] = __fadd_rn(acc[2], bf16lo(v.y));
  acc[3] = __fadd_rn(acc[3], bf16hi(v.y));
  acc[4] = __fadd_rn(acc[4], bf16lo(v.z));
  acc[5] = __fadd_rn(acc[5], bf16hi(v.z));
  acc[6] = __fadd_rn(acc[6], bf16lo(v.w));
  acc[7] = __fadd_rn(acc[7], bf16hi(v.w));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int CPT>
__global__ void __launch_bounds__(kThreads)
    combine_kernel(const char* __restrict__ y, const int32_t* __restrict__ dst_pos,
                   const float* __restrict__ gates, const char* __restrict__ shared,
                   const char* __restrict__ residual, int T, int H, int k, int64_t N,
                   char* __restrict__ out, WsHeader* hdr) {
  const int C8 = H >> 3;
  const int G = (C8 + CPT - 1) / CPT;
  const int64_t units = (int64_t)T * G;
  const size_t row_bytes = (size_t)H * 2;
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * kThreads) {
    const int t = (int)(u / G);
    const int g = (int)(u - (int64_t)t * G);
    float acc[CPT][8];
#pragma unroll
    for (int i = 0; i < CPT; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[i][e] = 0.0f;

    const int32_t* dp = dst_pos + (size_t)t * k;
    const float* gp = gates + (size_t)t * k;
    for (int j0 = 0; j0 < k; j0 += kBatch) {
      uint4 v[kBatch][CPT];
      float gw[kBatch];
      bool use[kBatch];
#pragma unroll
      for (int jj = 0; jj < kBatch; ++jj) {
        const int j = j0 + jj;
        int p = -1;
        gw[jj] = 0.0f;
        if (j < k) {
          p = __ldg(dp + j);
          gw[jj] = __ldg(gp + j);
          if (p >= N) {
            if (g == 0) report(hdr, MOE_ERR_DEVICE_RANGE, p);
            p = -1;
          }
        }
        use[jj] = p >= 0;
        const char* src = y + (size_t)(p < 0 ? 0 : p) * row_bytes;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
          const int c = g + i * G;
          if (use[jj] && c < C8)
            v[jj][i] = ld16_stream(src + (size_t)c * 16);
          else
            v[jj][i] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int jj = 0; jj < kBatch; ++jj)
        if (use[jj]) {
#pragma unroll
          for (int i = 0; i < CPT; ++i) fma8(acc[i], gw[jj], v[jj][i]);
        }
    }

#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = g + i * G;
      if (c >= C8) continue;
      const size_t off = (size_t)t * row_bytes + (size_t)c * 16;
      if (shared != nullptr) add8(acc[i], ld16_stream(shared + off));
      if (residual != nullptr) add8(acc[i], ld16_stream(residual + off));
      uint4 o;
      o.x = pack_bf16x2(acc[i][0], acc[i][1]);
      o.y = pack_bf16x2(acc[i][2], acc[i][3]);
      o.z = pack_bf16x2(acc[i][4], acc[i][5]);
      o.w = pack_bf16x2(acc[i][6], acc[i][7]);
      st16(out + off, o);
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

cudaError_t launch_combine(const LaunchEnv& env, const void* y, const int32_t* dst_pos,
                           const float* gates, const void* shared, const void* residual, int T,
                           int H, int k, int64_t N, void* out, WsHeader* hdr) {
  if (T == 0) return cudaSuccess;
  const int C8 = H / 8;
  auto kern = combine_kernel<1>;
  const int grid = grid_for(kern, env, (int64_t)T * C8);
  kern<<<grid, kThreads, 0, env.stream>>>(
      static_cast<const char*>(y), dst_pos, gates, static_cast<const char*>(shared),
      static_cast<const char*>(residual), T, H, k, N, static_cast<char*>(out), hdr);
  return cudaGetLastError();
}

}  // namespace moe
