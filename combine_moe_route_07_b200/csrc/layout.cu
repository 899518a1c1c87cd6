// layout.cu -- steps 2 and 3: per-expert count histogram and the layout scan
// (optionally fused with step 1, the router).
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
// One cooperative kernel, one CTA per tile of TT tokens (all CTAs resident at
// once, so CTAs may wait on one another; every wait is bounded):
//
//  1. (fused variant) route the tile's tokens, one warp per token.
//  2. Per-warp histograms of the tile's expert ids over contiguous runs of
//     assignments (__match_any_sync; the run leader adds), summed into the
//     tile histogram.  No atomics, so no result depends on scheduling.
//  3. Decoupled lookback across tiles, per expert, in an expert-major table:
//     publish the tile's aggregate, read a window of 32 predecessors at once,
//     add back to the nearest inclusive prefix, publish the inclusive prefix.
//     Flag and value share one 32-bit word (flag in bits 30-31).
//  4. The CTA of the last tile holds the totals: counts, expert offsets
//     (segments rounded to `align`, or C rows each), rank offsets and kept
//     rows per rank; it publishes them and raises a ready flag.
//  5. Every CTA places its assignments: token-order rank inside the expert =
//     tile prefix + warp prefix + lane rank within the run; capacity mode
//     keeps ranks < C.  Writes dst_pos / src_idx and marks its share of the
//     padding rows -1.
//  6. Once every lookback is done, each CTA clears its table column; the last
//     CTA to finish resets the counters, leaving the workspace ready.
#include "common.cuh"
#include "kernels.h"
#include "route_core.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kWindow = 32;
constexpr int kUnroll = 4;
constexpr uint32_t kFlagAgg = 1u << 30;
constexpr uint32_t kFlagIncl = 2u << 30;
constexpr uint32_t kValMask = (1u << 30) - 1u;
constexpr unsigned kMaxSpins = 1u << 26;

struct LayoutParams {
  const int32_t* ids;  // [T,k]: input, or written by step 1 in the fused kernel
  int32_t* ids_out;    // fused: where step 1 writes the ids (same buffer)
  const float* logits;
  const float* bias;
  float* gates;
  int renorm;
  int T, k, E, R, capacity, align, B, TT;
  int64_t N;
  uint32_t* table;  // [E][B] lookback words
  WsHeader* hdr;
  int32_t* counts;
  int32_t* expert_off;
  int32_t* rank_off;
  int32_t* rank_counts;
  int32_t* dst_pos;
  int32_t* src_idx;
  uint64_t timeout_ns;
};

// Wait until the word at p carries a flag; after the time limit record
// MOE_ERR_DEVICE_TIMEOUT and return a placeholder inclusive 0.
__device__ __noinline__ uint32_t wait_word(const uint32_t* p, WsHeader* hdr, uint64_t timeout_ns,
                                           int who) {
  const uint64_t t0 = global_ns();
  for (unsigned it = 0; it < kMaxSpins; ++it) {
    const uint32_t w = ld_relaxed(p);
    if (w & ~kValMask) return w;
    if ((it & 15u) == 15u) {
      if (error_seen(hdr) == MOE_ERR_DEVICE_TIMEOUT) return kFlagIncl;
      if (global_ns() - t0 > timeout_ns) break;
    }
    __nanosleep(64);
  }
  report(hdr, MOE_ERR_DEVICE_TIMEOUT, who);
  return kFlagIncl;
}

// Wait until *p >= target; false (and MOE_ERR_DEVICE_TIMEOUT) after the limit.
__device__ __noinline__ bool wait_count(const uint32_t* p, uint32_t target, WsHeader* hdr,
                                        uint64_t timeout_ns, int who) {
  const uint64_t t0 = global_ns();
  for (unsigned it = 0; it < kMaxSpins; ++it) {
    if (ld_acquire(p) >= target) return true;
    if ((it & 15u) == 15u) {
      if (error_seen(hdr) == MOE_ERR_DEVICE_TIMEOUT) return false;
      if (global_ns() - t0 > timeout_ns) break;
    }
    __nanosleep(128);
  }
  report(hdr, MOE_ERR_DEVICE_TIMEOUT, who);
  return false;
}

// Exclusive prefix of tile vb for one expert: sum the predecessors' words from
// the nearest back to the first inclusive one, 32 loads in flight at a time.
__device__ uint32_t lookback(const uint32_t* col, int vb, WsHeader* hdr, uint64_t timeout_ns) {
  uint32_t excl = 0;
  for (int hi = vb - 1; hi >= 0; hi -= kWindow) {
    uint32_t w[kWindow];
#pragma unroll
    for (int i = 0; i < kWindow; ++i) w[i] = (hi - i >= 0) ? ld_relaxed(col + hi - i) : 0u;
    bool done = false;
#pragma unroll
    for (int i = 0; i < kWindow; ++i) {
      if (!done && hi - i >= 0) {
        uint32_t v = w[i];
        if ((v & ~kValMask) == 0u) v = wait_word(col + hi - i, hdr, timeout_ns, vb);
        excl += v & kValMask;
        done = (v & ~kValMask) == kFlagIncl;
      }
    }
    if (done) break;
  }
  return excl & kValMask;
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

template <int NK, bool ROUTE>
__global__ void __launch_bounds__(kThreads) layout_kernel(const LayoutParams P) {
  extern __shared__ int32_t smem[];
  const int E = P.E, k = P.k, C = P.capacity;
  int32_t* wh = smem;                // [kWarps][E] per-warp counts, then bases
  int32_t* tile = wh + kWarps * E;   // [E] tile histogram, then inclusive prefix
  int32_t* off = tile + E;           // [E+1] expert offsets
  int32_t* kept = off + E + 1;       // [E]
  __shared__ int32_t s_wtot[kWarps];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vb = blockIdx.x;
  const int t0 = min(P.T, vb * P.TT);
  const int t1 = min(P.T, t0 + P.TT);

  if constexpr (ROUTE) {
    float b[NK];
    load_bias<NK>(P.bias, E, lane, b);
    for (int t = t0 + w; t < t1; t += kWarps) {
      int e;
      float g;
      bool nan_key;
      route_token<NK>(P.logits + (size_t)t * E, b, E, k, P.renorm, lane, e, g, nan_key);
      if (nan_key && lane == 0) report(P.hdr, MOE_ERR_DEVICE_NAN, t);
      if (lane < k) {
        P.ids_out[(size_t)t * k + lane] = e;
        P.gates[(size_t)t * k + lane] = g;
      }
    }
  }
  for (int i = threadIdx.x; i < kWarps * E; i += kThreads) wh[i] = 0;
  __syncthreads();  // (fused) the tile's ids are written before anyone reads them

  // this warp's contiguous run of the tile's assignments
  const int64_t i0 = (int64_t)t0 * k, i1 = (int64_t)t1 * k;
  const int64_t chunk = (((i1 - i0) + kWarps - 1) / kWarps + 31) / 32 * 32;
  const int64_t s0 = min(i1, i0 + (int64_t)w * chunk);
  const int64_t s1 = min(i1, s0 + chunk);
  int32_t* my = wh + w * E;

  // pass 1: per-warp histogram
  for (int64_t base = s0; base < s1; base += 32 * kUnroll) {
    int ev[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + 32 * u + lane;
      ev[u] = (i < s1) ? P.ids[i] : -1;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + 32 * u + lane;
      if (base + 32 * u < s1) {
        const bool ok = (i < s1) && (unsigned)ev[u] < (unsigned)E;
        if (i < s1 && !ok) report(P.hdr, MOE_ERR_DEVICE_RANGE, (int)i);
        const unsigned active = __ballot_sync(kFull, ok);
        if (ok) {
          const unsigned peers = __match_any_sync(active, ev[u]);
          if (lane == __ffs(peers) - 1) my[ev[u]] += __popc(peers);
        }
        __syncwarp();
      }
    }
  }
  __syncthreads();

  // tile histogram; publish the aggregate (tile 0: its inclusive prefix)
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int h = 0;
    for (int q = 0; q < kWarps; ++q) h += wh[q * E + e];
    tile[e] = h;
    st_relaxed(P.table + (size_t)e * P.B + vb, (vb == 0 ? kFlagIncl : kFlagAgg) | (uint32_t)h);
  }
  // lookback; then each warp's first token-order rank in each expert
  for (int e = threadIdx.x; e < E; e += kThreads) {
    const uint32_t ex = (vb > 0) ? lookback(P.table + (size_t)e * P.B, vb, P.hdr, P.timeout_ns)
                                 : 0u;
    if (vb > 0)
      st_relaxed(P.table + (size_t)e * P.B + vb, kFlagIncl | ((ex + (uint32_t)tile[e]) & kValMask));
    int run = (int)ex;
    for (int q = 0; q < kWarps; ++q) {
      const int c = wh[q * E + e];
      wh[q * E + e] = run;
      run += c;
    }
    tile[e] = run;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(&P.hdr->looked, 1u);
  }

  // the last tile's inclusive prefixes are the totals
  if (vb == P.B - 1) {
    for (int e = threadIdx.x; e < E; e += kThreads) {
      const int c = tile[e];
      P.counts[e] = c;
      off[e] = C > 0 ? C : ((c + P.align - 1) / P.align) * P.align;
      kept[e] = (C > 0 && c > C) ? C : c;
    }
    __syncthreads();
    const int used = block_exclusive_scan(off, E, s_wtot);
    const int kept_total = block_exclusive_scan(kept, E, s_wtot);
    const int Er = E / P.R;
    for (int e = threadIdx.x; e < E; e += kThreads) P.expert_off[e] = off[e];
    for (int r = threadIdx.x; r < P.R; r += kThreads) {
      P.rank_off[r] = off[r * Er];
      const int hi = (r + 1 < P.R) ? kept[(r + 1) * Er] : kept_total;
      P.rank_counts[r] = hi - kept[r * Er];
    }
    if (threadIdx.x == 0) {
      P.expert_off[E] = used;
      P.rank_off[P.R] = used;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      st_release(&P.hdr->totals_ready, 1u);
    }
  }
  if (threadIdx.x == 0) wait_count(&P.hdr->totals_ready, 1u, P.hdr, P.timeout_ns, vb);
  __syncthreads();
  const bool fill = (C > 0 || P.align > 1);
  for (int e = threadIdx.x; e <= E; e += kThreads) off[e] = ld_cg(P.expert_off + e);
  if (fill)
    for (int e = threadIdx.x; e < E; e += kThreads) {
      const int c = ld_cg(P.counts + e);
      kept[e] = (C > 0 && c > C) ? C : c;
    }
  __syncthreads();

  // pass 2: place each assignment at its token-order rank
  for (int64_t base = s0; base < s1; base += 32 * kUnroll) {
    int ev[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + 32 * u + lane;
      ev[u] = (i < s1) ? P.ids[i] : -1;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + 32 * u + lane;
      if (base + 32 * u < s1) {
        const int e = ev[u];
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
          int64_t dst = -1;
          if (ok) dst = (C > 0) ? (v < C ? (int64_t)e * C + v : -1) : (int64_t)off[e] + v;
          // in range by construction; checked because a lookback that gave up
          // leaves placeholder prefixes
          if (dst >= P.N || (ok && v < 0)) {
            report(P.hdr, MOE_ERR_DEVICE_RANGE, (int)dst);
            dst = -1;
          }
          P.dst_pos[i] = (int32_t)dst;
          if (dst >= 0) P.src_idx[dst] = (int32_t)i;
        }
      }
    }
  }

  // rows that hold no assignment (alignment padding, unused capacity slots)
  if (fill) {
    const int64_t per = (P.N + P.B - 1) / P.B;
    const int64_t r0 = (int64_t)vb * per;
    const int64_t r1 = min(P.N, r0 + per);
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
      if (pad) P.src_idx[p] = -1;
    }
  }

  // once no lookback reads the table any more, clear this tile's column
  if (threadIdx.x == 0) wait_count(&P.hdr->looked, (uint32_t)P.B, P.hdr, P.timeout_ns, vb);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads) P.table[(size_t)e * P.B + vb] = 0u;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&P.hdr->finished, 1u) == (uint32_t)P.B - 1u) {
      P.hdr->looked = 0u;
      P.hdr->totals_ready = 0u;
      P.hdr->finished = 0u;
    }
  }
}

template <int NK, bool ROUTE>
cudaError_t launch_fused(const LaunchEnv& env, LayoutParams P) {
  auto kern = layout_kernel<NK, ROUTE>;
  const size_t smem = (11 * (size_t)P.E + 1) * sizeof(int32_t);
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t max_blocks = (int64_t)per_sm * env.num_sms;
  // tiles of 128 tokens, doubled until every tile's CTA can be resident at once
  int64_t TT = kLayoutTileTokens;
  int64_t B = P.T > 0 ? (P.T + TT - 1) / TT : 1;
  while (B > max_blocks) {
    TT *= 2;
    B = (P.T + TT - 1) / TT;
  }
  P.TT = (int)TT;
  P.B = (int)B;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = env.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

}  // namespace

cudaError_t launch_layout(const LaunchEnv& env, const int32_t* ids, int T, int E, int k, int R,
                          int capacity, int align, int64_t N, uint32_t* table, WsHeader* hdr,
                          int32_t* counts, int32_t* expert_off, int32_t* rank_off,
                          int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx,
                          uint64_t timeout_ns) {
  LayoutParams P{};
  P.ids = ids;
  P.T = T;
  P.k = k;
  P.E = E;
  P.R = R;
  P.capacity = capacity;
  P.align = align;
  P.N = N;
  P.table = table;
  P.hdr = hdr;
  P.counts = counts;
  P.expert_off = expert_off;
  P.rank_off = rank_off;
  P.rank_counts = rank_counts;
  P.dst_pos = dst_pos;
  P.src_idx = src_idx;
  P.timeout_ns = timeout_ns;
  return launch_fused<1, false>(env, P);
}

cudaError_t launch_route_layout(const LaunchEnv& env, const float* logits, const float* bias,
                                int renorm, int32_t* ids, float* gates, int T, int E, int k,
                                int R, int capacity, int align, int64_t N, uint32_t* table,
                                WsHeader* hdr, int32_t* counts, int32_t* expert_off,
                                int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                                int32_t* src_idx, uint64_t timeout_ns) {
  LayoutParams P{};
  P.ids = ids;
  P.ids_out = ids;
  P.logits = logits;
  P.bias = bias;
  P.gates = gates;
  P.renorm = renorm;
  P.T = T;
  P.k = k;
  P.E = E;
  P.R = R;
  P.capacity = capacity;
  P.align = align;
  P.N = N;
  P.table = table;
  P.hdr = hdr;
  P.counts = counts;
  P.expert_off = expert_off;
  P.rank_off = rank_off;
  P.rank_counts = rank_counts;
  P.dst_pos = dst_pos;
  P.src_idx = src_idx;
  P.timeout_ns = timeout_ns;
  const int nk = (E + 31) / 32;
  if (nk <= 1) return launch_fused<1, true>(env, P);
  if (nk <= 2) return launch_fused<2, true>(env, P);
  if (nk <= 4) return launch_fused<4, true>(env, P);
  if (nk <= 8) return launch_fused<8, true>(env, P);
  if (nk <= 16) return launch_fused<16, true>(env, P);
  return launch_fused<32, true>(env, P);
}

}  // namespace moe
