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
// Token-major gather, HBM-bound.  Each warp owns a 32*CPT-chunk slice of one
// token row; each lane issues the 16-byte loads of up to kBatch slots before
// using any of them (independent loads in flight), then accumulates in fp32
// in slot order j = 0..k-1 with explicit round-to-nearest FMAs, adds the
// shared-expert row and the residual row, and rounds to bf16 once.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 256;


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

// One warp per (token, slice of 32*CPT chunks); lane j < k fetches the row
// and gate of slot j once and the warp broadcasts them by shuffle.  With
// PF the next task's rows and gates are fetched while this one computes, and
// a batch of slots that are all dropped issues no loads at all (capacity mode
// drops most slots of a skewed batch).
template <int CPT, int KB, int MINB, bool PF>
__global__ void __launch_bounds__(kThreads, MINB)
    combine_kernel(const char* __restrict__ y, const int32_t* __restrict__ dst_pos,
                   const float* __restrict__ gates, const char* __restrict__ shared,
                   const char* __restrict__ residual, int T, int H, int k, int64_t N,
                   char* __restrict__ out, WsHeader* hdr) {
  pdl_wait();  // y, gates and dst_pos may come from the kernel launched just before
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int C8 = H >> 3;
  const int S = (C8 + 32 * CPT - 1) / (32 * CPT);
  const int64_t tasks = (int64_t)T * S;
  const size_t row_bytes = (size_t)H * 2;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
  // slot j of task `task` (lane j < k), -1 when dropped or out of range
  auto fetch = [&](int64_t task, int& p, float& g) {
    p = -1;
    g = 0.0f;
    if (task < tasks && lane < k) {
      const int t = (int)((uint32_t)task / (uint32_t)S);  // tasks < 2^31 (host check)
      p = __ldg(dst_pos + (size_t)t * k + lane);
      g = __ldg(gates + (size_t)t * k + lane);
      if (p >= N) {
        report(hdr, MOE_ERR_DEVICE_RANGE, p);
        p = -1;
      }
    }
  };
  int64_t task = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  int pl, pn = -1;
  float gl, gn = 0.0f;
  fetch(task, pl, gl);
  for (; task < tasks; task += nw) {
    if (PF) fetch(task + nw, pn, gn);
    const int t = (int)((uint32_t)task / (uint32_t)S);
    const int cb = (int)((uint32_t)task - (uint32_t)t * (uint32_t)S) * 32 * CPT + lane;
    const unsigned kept = __ballot_sync(kFull, pl >= 0);
    float acc[CPT][8];
#pragma unroll
    for (int i = 0; i < CPT; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[i][e] = 0.0f;

    for (int j0 = 0; j0 < k; j0 += KB) {
      if (((kept >> j0) & ((1u << KB) - 1u)) == 0u) continue;  // every slot dropped
      uint4 v[KB][CPT];
      float gw[KB];
      int pp[KB];
#pragma unroll
      for (int jj = 0; jj < KB; ++jj) {
        const int j = j0 + jj;  // j < 32: the shuffle source is always a lane
        pp[jj] = __shfl_sync(kFull, pl, j & 31);
        gw[jj] = __shfl_sync(kFull, gl, j & 31);
        if (j >= k) pp[jj] = -1;
        const char* src = y + (size_t)(pp[jj] < 0 ? 0 : pp[jj]) * row_bytes;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
          const int c = cb + 32 * i;
          if (pp[jj] >= 0 && c < C8)
            v[jj][i] = ld16_stream(src + (size_t)c * 16);
          else
            v[jj][i] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int jj = 0; jj < KB; ++jj)
        if (pp[jj] >= 0) {
#pragma unroll
          for (int i = 0; i < CPT; ++i) fma8(acc[i], gw[jj], v[jj][i]);
        }
    }

#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = cb + 32 * i;
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
    if (PF) {
      pl = pn;
      gl = gn;
    } else {
      fetch(task + nw, pl, gl);
    }
  }
}

// Enough CTAs for one warp per task, at most the ones resident at once.
template <typename K>
int grid_for(K kernel, const LaunchEnv& env, int64_t tasks) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t need = (tasks + kThreads / 32 - 1) / (kThreads / 32);
  const int64_t cap = (int64_t)env.num_sms * per_sm;
  int64_t g = need < cap ? need : cap;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_combine(const LaunchEnv& env, const void* y, const int32_t* dst_pos,
                           const float* gates, const void* shared, const void* residual, int T,
                           int H, int k, int64_t N, void* out, WsHeader* hdr, bool sparse) {
  if (T == 0) return cudaSuccess;
  const int C8 = H / 8;
  const char* ys = static_cast<const char*>(y);
  const char* sh = static_cast<const char*>(shared);
  const char* rs = static_cast<const char*>(residual);
  char* o = static_cast<char*>(out);
  // Capacity mode drops most slots of a skewed batch: then each task moves
  // little and its latency dominates, so wider slices with the next task's
  // metadata prefetched win; dense layouts do better with more warps.
  if (sparse && C8 >= 128) {
    auto kern = combine_kernel<4, 2, 2, true>;
    const int grid = grid_for(kern, env, (int64_t)T * ((C8 + 127) / 128));
    return launch_pdl(env, kern, dim3(grid), dim3(kThreads), 0, ys, dst_pos, gates, sh, rs, T, H,
                      k, N, o, hdr);
  }
  auto kern = combine_kernel<1, 4, 4, false>;
  const int grid = grid_for(kern, env, (int64_t)T * ((C8 + 31) / 32));
  return launch_pdl(env, kern, dim3(grid), dim3(kThreads), 0, ys, dst_pos, gates, sh, rs, T, H, k,
                    N, o, hdr);
}

}  // namespace moe
