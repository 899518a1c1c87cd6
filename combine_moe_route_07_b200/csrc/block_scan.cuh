// block_scan.cuh -- exclusive prefix sum over a shared-memory array by one
// CTA (used by the layout kernels to turn per-expert row counts into segment
// offsets).
#pragma once

#include "common.cuh"

namespace moe {

// Exclusive scan of v[0..n) in shared memory by the whole CTA (n <= 4 *
// THREADS).  Returns the total to every thread.
template <int THREADS>
__device__ int block_exclusive_scan(int32_t* v, int n, int32_t* warp_tot) {
  constexpr int kW = THREADS / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int per = (n + THREADS - 1) / THREADS;
  const int lo = threadIdx.x * per;
  int local = 0;
  for (int i = 0; i < per; ++i)
    if (lo + i < n) local += v[lo + i];
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = (lane < kW) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kW) warp_tot[lane] = s;
  }
  __syncthreads();
  int run = (wid > 0 ? warp_tot[wid - 1] : 0) + x - local;
  const int total = warp_tot[kW - 1];
  for (int i = 0; i < per; ++i)
    if (lo + i < n) {
      const int t = v[lo + i];
      v[lo + i] = run;
      run += t;
    }
  __syncthreads();
  return total;
}

}  // namespace moe
