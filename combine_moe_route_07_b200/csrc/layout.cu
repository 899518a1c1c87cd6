// layout.cu -- steps 2 and 3: per-expert count histogram and the layout scan.
//
// "GPU MoE all-to-all" (aicassindra), section "Two collectives per layer":
// per-destination counts precede the payload; section "Bucketing": sort rows
// by destination, build the offset table, keep indices and counts on the
// device.  "MoE All-to-All Dispatch and Ragged Routing", section "Fixed
// Capacity vs. Ragged Routing": rigid per-expert slots with drops, or a
// dropless ragged layout.  "Mixture-of-experts acceleration through overlap":
// each destination's rows form one contiguous band (experts are numbered
// rank-major, so rank slices are unions of consecutive expert segments).
//
// Two kernels over tiles of kLayoutTileTokens tokens:
//
//  count  one CTA per tile, virtual tile id from an atomic ticket (so every
//         tile a CTA waits on belongs to a CTA that is already running).
//         Shared-memory histogram of the tile's expert ids, then a
//         decoupled-lookback scan across tiles, per expert: publish the
//         tile's aggregate, walk back over predecessors until an inclusive
//         prefix is found, publish the inclusive prefix.  Flag and value
//         share one 32-bit word (flag in bits 30-31), so a relaxed store is
//         enough.  The CTA holding the last tile sees the totals and writes
//         counts, expert/rank offsets and per-rank kept counts.
//  place  one CTA per tile again.  Warps own contiguous runs of the tile's
//         assignments; per-warp histograms (__match_any_sync, leader adds)
//         and a scan over warps give each assignment its token-order rank
//         inside its expert with no atomics, so the result never depends on
//         scheduling.  Writes dst_pos / src_idx, marks padding rows -1 and
//         leaves the lookback table and ticket zeroed for the next call.
//
// Every wait is bounded: after `timeout_ns` it records
// MOE_ERR_DEVICE_TIMEOUT, publishes a placeholder so successors stop
// waiting, and returns.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kFlagAgg = 1u << 30;
constexpr uint32_t kFlagIncl = 2u << 30;
constexpr uint32_t kValMask = (1u << 30) - 1u;
constexpr unsigned kMaxSpins = 1u << 26;

__device__ uint32_t wait_published(const uint32_t* p, WsHeader* hdr, uint64_t timeout_ns,
                                   int who) {
  uint32_t w = ld_relaxed(p);
  if (w & ~kValMask) return w;
  const uint64_t t0 = global_ns();
  for (unsigned it = 1; it < kMaxSpins; ++it) {
    __nanosleep(64);
    w = ld_relaxed(p);
    if (w & ~kValMask) return w;
    if ((it & 15u) == 0u) {
      if (error_seen(hdr) == MOE_ERR_DEVICE_TIMEOUT) return kFlagIncl;
      if (global_ns() - t0 > timeout_ns) break;
    }
  }
  report(hdr, MOE_ERR_DEVICE_TIMEOUT, who);
  return kFlagIncl;
}

// Exclusive scan of v[0..n) in shared memory by the whole CTA (n <= 4 *
// kThreads).  Returns the total to every thread.
__device__ int block_exclusive_scan(int32_t* v, int n, int32_t* warp_tot) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int per = (n + kThreads - 1) / kThreads;
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
    int s = (lane < kWarps) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kWarps) warp_tot[lane] = s;
  }
  __syncthreads();
  int run = (wid > 0 ? warp_tot[wid - 1] : 0) + x - local;
  const int total = warp_tot[kWarps - 1];
  for (int i = 0; i < per; ++i)
    if (lo + i < n) {
      const int t = v[lo + i];
      v[lo + i] = run;
      run += t;
    }
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kThreads)
    layout_count_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int R, int capacity,
                        int align, int B, uint32_t* __restrict__ status, WsHeader* hdr,
                        int32_t* __restrict__ counts, int32_t* __restrict__ expert_off,
                        int32_t* __restrict__ rank_off, int32_t* __restrict__ rank_counts,
                        uint64_t timeout_ns) {
  extern __shared__ int32_t smem[];
  int32_t* hist = smem;     // [E] this tile's histogram, later the segment scan
  int32_t* tot = smem + E;  // [E] inclusive prefix through this tile
  __shared__ uint32_t s_vb;
  __shared__ int32_t s_wtot[kWarps];

  if (threadIdx.x == 0) s_vb = atomicAdd(&hdr->ticket, 1u);
  for (int e = threadIdx.x; e < E; e += kThreads) hist[e] = 0;
  __syncthreads();
  const int vb = (int)s_vb;
  if (vb >= B) {  // only with a workspace that was not left zeroed
    if (threadIdx.x == 0) report(hdr, MOE_ERR_WORKSPACE, vb);
    return;
  }

  const int64_t i0 = (int64_t)vb * kLayoutTileTokens * k;
  const int64_t i1 = (int64_t)min(T, (vb + 1) * kLayoutTileTokens) * k;
  for (int64_t i = i0 + threadIdx.x; i < i1; i += kThreads) {
    const int e = __ldg(ids + i);
    if ((unsigned)e < (unsigned)E)
      atomicAdd(&hist[e], 1);
    else
      report(hdr, MOE_ERR_DEVICE_RANGE, (int)i);
  }
  __syncthreads();

  uint32_t* mine = status + (size_t)vb * E;
  const uint32_t flag0 = (vb == 0) ? kFlagIncl : kFlagAgg;
  for (int e = threadIdx.x; e < E; e += kThreads) st_relaxed(mine + e, flag0 | (uint32_t)hist[e]);

  for (int e = threadIdx.x; e < E; e += kThreads) {
    uint32_t excl = 0;
    for (int p = vb - 1; p >= 0; --p) {
      const uint32_t w = wait_published(status + (size_t)p * E + e, hdr, timeout_ns, vb);
      excl += w & kValMask;
      if ((w & ~kValMask) == kFlagIncl) break;
    }
    const uint32_t incl = (excl + (uint32_t)hist[e]) & kValMask;
    if (vb > 0) st_relaxed(mine + e, kFlagIncl | incl);
    tot[e] = (int32_t)incl;
  }

  if (vb != B - 1) return;
  // The last tile's inclusive prefixes are the totals.
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads) {
    const int c = tot[e];
    counts[e] = c;
    hist[e] = capacity > 0 ? capacity : ((c + align - 1) / align) * align;
    tot[e] = (capacity > 0 && c > capacity) ? capacity : c;  // kept
  }
  __syncthreads();
  const int used = block_exclusive_scan(hist, E, s_wtot);
  const int kept_total = block_exclusive_scan(tot, E, s_wtot);
  for (int e = threadIdx.x; e < E; e += kThreads) expert_off[e] = hist[e];
  const int Er = E / R;
  for (int r = threadIdx.x; r < R; r += kThreads) {
    rank_off[r] = hist[r * Er];
    const int hi = (r + 1 < R) ? tot[(r + 1) * Er] : kept_total;
    rank_counts[r] = hi - tot[r * Er];
  }
  if (threadIdx.x == 0) {
    expert_off[E] = used;
    rank_off[R] = used;
  }
}

__global__ void __launch_bounds__(kThreads)
    layout_place_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int capacity, int B,
                        int64_t N, int fill, uint32_t* __restrict__ status, WsHeader* hdr,
                        const int32_t* __restrict__ counts, const int32_t* __restrict__ expert_off,
                        int32_t* __restrict__ dst_pos, int32_t* __restrict__ src_idx) {
  extern __shared__ int32_t smem[];
  int32_t* wh = smem;                // [kWarps][E] per-warp counters
  int32_t* off = smem + kWarps * E;  // [E+1]  (padding fill)
  int32_t* kept = off + E + 1;       // [E]
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;

  if (b == 0 && threadIdx.x == 0) hdr->ticket = 0u;  // the count pass is over
  for (int i = threadIdx.x; i < kWarps * E; i += kThreads) wh[i] = 0;
  __syncthreads();

  const int64_t i0 = (int64_t)b * kLayoutTileTokens * k;
  const int64_t i1 = (int64_t)min(T, (b + 1) * kLayoutTileTokens) * k;
  const int64_t n = i1 - i0;
  const int64_t chunk = (((n + kWarps - 1) / kWarps) + 31) / 32 * 32;
  const int64_t s0 = min(i1, i0 + (int64_t)w * chunk);
  const int64_t s1 = min(i1, s0 + chunk);
  int32_t* my = wh + w * E;

  // pass 1: per-warp histogram of this warp's run
  for (int64_t base = s0; base < s1; base += 32) {
    const int64_t i = base + lane;
    const int e = (i < s1) ? __ldg(ids + i) : -1;
    const bool ok = (i < s1) && (unsigned)e < (unsigned)E;
    const unsigned active = __ballot_sync(kFull, ok);
    if (ok) {
      const unsigned peers = __match_any_sync(active, e);
      if (lane == __ffs(peers) - 1) my[e] += __popc(peers);
    }
    __syncwarp();
  }
  __syncthreads();

  // first row (dropless) or first token-order rank (capacity) of each warp's
  // share of each expert
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int h = 0;
    for (int q = 0; q < kWarps; ++q) h += wh[q * E + e];
    const int incl = (int)(status[(size_t)b * E + e] & kValMask);
    int run = (capacity > 0 ? 0 : expert_off[e]) + (incl - h);
    for (int q = 0; q < kWarps; ++q) {
      const int c = wh[q * E + e];
      wh[q * E + e] = run;
      run += c;
    }
    status[(size_t)b * E + e] = 0u;
  }
  __syncthreads();

  // pass 2: rank inside the warp's step, in lane (= token) order
  for (int64_t base = s0; base < s1; base += 32) {
    const int64_t i = base + lane;
    const int e = (i < s1) ? __ldg(ids + i) : -1;
    const bool ok = (i < s1) && (unsigned)e < (unsigned)E;
    const unsigned active = __ballot_sync(kFull, ok);
    int v = 0, cnt = 0;
    bool lead = false;
    if (ok) {
      const unsigned peers = __match_any_sync(active, e);
      v = my[e] + __popc(peers & lanemask_lt());
      lead = (lane == __ffs(peers) - 1);
      cnt = __popc(peers);
    }
    __syncwarp();
    if (lead) my[e] = v + cnt;
    __syncwarp();
    if (i < s1) {
      int dst = -1;
      if (ok) dst = (capacity > 0) ? (v < capacity ? e * capacity + v : -1) : v;
      // Positions are in range by construction; the check only matters after
      // a count pass that gave up (its prefixes are placeholders).
      if (dst >= N || (ok && v < 0)) {
        report(hdr, MOE_ERR_DEVICE_RANGE, dst);
        dst = -1;
      }
      dst_pos[i] = dst;
      if (dst >= 0) src_idx[dst] = (int32_t)i;
    }
  }

  if (!fill) return;
  // rows that hold no assignment: alignment padding, unused capacity slots
  for (int e = threadIdx.x; e <= E; e += kThreads) off[e] = expert_off[e];
  for (int e = threadIdx.x; e < E; e += kThreads) {
    const int c = counts[e];
    kept[e] = (capacity > 0 && c > capacity) ? capacity : c;
  }
  __syncthreads();
  const int64_t per = (N + B - 1) / B;
  const int64_t r0 = (int64_t)b * per;
  const int64_t r1 = min(N, r0 + per);
  for (int64_t p = r0 + threadIdx.x; p < r1; p += kThreads) {
    bool pad = true;
    if (p < off[E]) {
      int lo = 0, hi = E - 1;  // last e with off[e] <= p
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= p)
          lo = mid;
        else
          hi = mid - 1;
      }
      pad = (p - off[lo]) >= kept[lo];
    }
    if (pad) src_idx[p] = -1;
  }
}

}  // namespace

cudaError_t launch_layout(const LaunchEnv& env, const int32_t* ids, int T, int E, int k, int R,
                          int capacity, int align, int64_t N, uint32_t* status, WsHeader* hdr,
                          int32_t* counts, int32_t* expert_off, int32_t* rank_off,
                          int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx,
                          uint64_t timeout_ns) {
  const int B = T > 0 ? (T + kLayoutTileTokens - 1) / kLayoutTileTokens : 1;
  const size_t smem_count = (size_t)2 * E * sizeof(int32_t);
  layout_count_kernel<<<B, kThreads, smem_count, env.stream>>>(
      ids, T, k, E, R, capacity, align, B, status, hdr, counts, expert_off, rank_off, rank_counts,
      timeout_ns);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int fill = (capacity > 0 || align > 1) ? 1 : 0;
  const size_t smem_place = ((size_t)kWarps * E + 2 * (size_t)E + 1) * sizeof(int32_t);
  layout_place_kernel<<<B, kThreads, smem_place, env.stream>>>(
      ids, T, k, E, capacity, B, N, fill, status, hdr, counts, expert_off, dst_pos, src_idx);
  return cudaGetLastError();
}

}  // namespace moe
