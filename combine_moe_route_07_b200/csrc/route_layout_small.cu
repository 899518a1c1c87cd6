// route_layout_small.cu -- steps 1-3 for a small (decode-sized) batch in
// ONE launch: a thread-block cluster whose CTAs share their histograms
// through distributed shared memory.
//
// "GPU MoE all-to-all" (aicassindra), section "Latency-bound at decode,
// bandwidth-bound at prefill": at decode the exchange is latency-bound, so
// the metadata step must not add round trips.  With T*k small, a cluster of
// kClusterCtas CTAs routes the batch (CTA c the c-th contiguous block of
// tokens, one warp per token, the same selection code as route.cu), each CTA
// counts its ids in its own shared memory, one cluster barrier later every
// CTA reads all the CTAs' counts over DSMEM (totals, and its prefix from the
// earlier CTAs), scans the expert offsets, ranks its own assignments in
// token order and places them.  No tile table in global memory, no second
// launch.  The results are the same bits as route + count + place.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "route_core.cuh"

namespace moe {

namespace {

namespace cg = cooperative_groups;

constexpr int kSmallThreads = 512;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kClusterCtas = 8;  // portable cluster size

struct SmallParams {
  const float* logits;
  const float* bias;
  int T, E, k, R, renorm, capacity, align;
  int64_t N;
  WsHeader* hdr;
  int32_t* ids;
  float* gates;
  int32_t* counts;
  int32_t* expert_off;
  int32_t* rank_off;
  int32_t* rank_counts;
  int32_t* dst_pos;
  int32_t* src_idx;
};

// Exclusive scan of v[0..n) (n <= kSmallThreads) in place; returns the total.
// Starts and ends with a CTA barrier.
__device__ int small_scan(int32_t* v, int n, int32_t* wtot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  __syncthreads();
  const int x0 = threadIdx.x < n ? v[threadIdx.x] : 0;
  int x = x0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wtot[w] = x;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int q = 0; q < kSmallWarps; ++q) {
    if (q < w) before += wtot[q];
    total += wtot[q];
  }
  __syncthreads();
  if (threadIdx.x < n) v[threadIdx.x] = before + x - x0;
  __syncthreads();
  return total;
}

template <int NK>
__global__ void __launch_bounds__(kSmallThreads, 1) route_layout_small_kernel(const SmallParams P) {
  // dynamic: hist[E] this CTA's counts, pre[E] earlier CTAs' counts, off[E+1],
  // kept[E], wh[kSmallWarps][E] per-warp counts then bases, sid[TB*k] ids,
  // srk[TB*k] ranks in the warp's run
  extern __shared__ int32_t sm[];
  __shared__ __align__(16) uint32_t cand_all[kSmallWarps][NK >= 8 ? 3 * kMaxCand : 1];
  __shared__ int32_t wtot[kSmallWarps];
  cg::cluster_group cluster = cg::this_cluster();
  const int T = P.T, E = P.E, k = P.k, C = P.capacity;
  const int c = (int)cluster.block_rank();
  const int TB = (T + kClusterCtas - 1) / kClusterCtas;  // tokens per CTA
  const int t0 = min(T, c * TB), t1 = min(T, t0 + TB);
  const int n = (t1 - t0) * k;  // this CTA's assignments, from t0 * k
  int32_t* hist = sm;
  int32_t* pre = hist + E;
  int32_t* off = pre + E;
  int32_t* kept = off + E + 1;
  int32_t* wh = kept + E;
  int32_t* sid = wh + kSmallWarps * E;
  int32_t* srk = sid + TB * k;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  pdl_wait();  // logits may come from the kernel launched just before
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += kSmallThreads) hist[e] = 0;
  for (int x = threadIdx.x; x < kSmallWarps * E; x += kSmallThreads) wh[x] = 0;
  float b[NK];
  load_bias<NK>(P.bias, E, lane, b);
  __syncthreads();

  // 1. route this CTA's tokens, one warp per token
  for (int t = t0 + w; t < t1; t += kSmallWarps) {
    int e1 = 0;
    float g1 = 0.0f;
    int nan_tok;
    if constexpr (NK >= 8) {
      nan_tok = route_token_thr<NK>(P.logits, t, T, b, E, k, P.renorm, lane, cand_all[w], e1,
                                    g1);
    } else {
      int tok[1] = {t}, ea[1];
      float ga[1];
      nan_tok = route_tokens<NK, 1>(P.logits, tok, T, b, E, k, P.renorm, lane, ea, ga);
      e1 = ea[0];
      g1 = ga[0];
    }
    if (nan_tok >= 0 && lane == 0) report(P.hdr, MOE_ERR_DEVICE_NAN, nan_tok);
    if (lane < k) {
      P.ids[(size_t)t * k + lane] = e1;
      P.gates[(size_t)t * k + lane] = g1;
      sid[(t - t0) * k + lane] = e1;
      atomicAdd(&hist[e1], 1);
    }
  }
  cluster.sync();  // every CTA's counts are complete and visible to the cluster

  // 2. totals and the earlier CTAs' counts, read over DSMEM
  for (int e = threadIdx.x; e < E; e += kSmallThreads) {
    int tot = 0, before = 0;
#pragma unroll
    for (int q = 0; q < kClusterCtas; ++q) {
      const int v = cluster.map_shared_rank(hist, q)[e];
      tot += v;
      if (q < c) before += v;
    }
    pre[e] = before;
    off[e] = C > 0 ? C : ((tot + P.align - 1) / P.align) * P.align;
    kept[e] = (C > 0 && tot > C) ? C : tot;
    if (c == 0) P.counts[e] = tot;
  }
  cluster.sync();  // no CTA leaves while another still reads its counts
  const int used = small_scan(off, E, wtot);  // (synchronises the CTA)
  if (threadIdx.x == 0) off[E] = used;
  __syncthreads();
  if (c == 0) {
    const int Er = E / P.R;
    for (int e = threadIdx.x; e <= E; e += kSmallThreads) P.expert_off[e] = off[e];
    for (int r = w; r < P.R; r += kSmallWarps) {  // one warp per rank: rows kept
      int s = 0;
      for (int e = r * Er + lane; e < (r + 1) * Er; e += 32) s += kept[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
      if (lane == 0) {
        P.rank_counts[r] = s;
        P.rank_off[r] = off[r * Er];
      }
    }
    if (threadIdx.x == 0) P.rank_off[P.R] = used;
  }

  // 3. token-order ranks of this CTA's assignments: warp w a contiguous run
  const int chunk = ((n + kSmallWarps - 1) / kSmallWarps + 31) / 32 * 32;
  const int s0 = min(n, w * chunk), s1 = min(n, s0 + chunk);
  int32_t* my = wh + w * E;
  for (int r0 = s0; r0 < s1; r0 += 32) {
    const int i = r0 + lane;
    const bool ok = i < s1;
    const int e = ok ? sid[i] : -1;
    const unsigned active = __ballot_sync(kFull, ok);
    if (ok) {
      const unsigned peers = __match_any_sync(active, e);
      const int v = my[e] + __popc(peers & lanemask_lt());
      __syncwarp(active);
      if (lane == __ffs(peers) - 1) my[e] = v + __popc(peers);
      srk[i] = v;
    }
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kSmallThreads) {  // warp counts -> bases
    int acc = pre[e];
    for (int q = 0; q < kSmallWarps; ++q) {
      const int v = wh[q * E + e];
      wh[q * E + e] = acc;
      acc += v;
    }
  }
  __syncthreads();

  // 4. place this CTA's assignments
  for (int i = threadIdx.x; i < n; i += kSmallThreads) {
    const int e = sid[i];
    const int rank = wh[(i / chunk) * E + e] + srk[i];
    const int64_t dst = (C > 0 && rank >= C) ? -1 : (int64_t)off[e] + rank;
    P.dst_pos[(size_t)t0 * k + i] = (int32_t)dst;
    if (dst >= 0) P.src_idx[dst] = t0 * k + i;
  }
  // 5. rows without an assignment (alignment padding, unused capacity slots),
  //    split over the cluster's CTAs
  if (C > 0 || P.align > 1) {
    const int64_t per = (P.N + kClusterCtas - 1) / kClusterCtas;
    const int64_t r0 = (int64_t)c * per, r1 = min(P.N, r0 + per);
    for (int64_t p = r0 + threadIdx.x; p < r1; p += kSmallThreads) {
      bool pad = true;
      if (p < used) {
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
}

template <int NK>
cudaError_t launch_small(const LaunchEnv& env, const SmallParams& P) {
  const int TB = (P.T + kClusterCtas - 1) / kClusterCtas;
  const size_t smem = ((size_t)4 * P.E + 1 + (size_t)kSmallWarps * P.E + (size_t)2 * TB * P.k) *
                      sizeof(int32_t);
  auto kern = route_layout_small_kernel<NK>;
  int per_sm = 1;  // (raises the kernel's dynamic shared-memory limit to smem)
  cudaError_t err =
      blocks_per_sm(reinterpret_cast<const void*>(kern), kSmallThreads, smem, &per_sm);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kClusterCtas);
  cfg.blockDim = dim3(kSmallThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = env.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClusterCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

}  // namespace

bool route_layout_small_fits(int T, int E, int k) {
  return T > 0 && E <= kSmallMaxExperts && (int64_t)T * k <= kSmallMaxAssign;
}

cudaError_t launch_route_layout_small(const LaunchEnv& env, const float* logits,
                                      const float* bias, int T, int E, int k, int R, int renorm,
                                      int capacity, int align, int64_t N, WsHeader* hdr,
                                      int32_t* ids, float* gates, int32_t* counts,
                                      int32_t* expert_off, int32_t* rank_off,
                                      int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx) {
  SmallParams P;
  P.logits = logits;
  P.bias = bias;
  P.T = T;
  P.E = E;
  P.k = k;
  P.R = R;
  P.renorm = renorm;
  P.capacity = capacity;
  P.align = align;
  P.N = N;
  P.hdr = hdr;
  P.ids = ids;
  P.gates = gates;
  P.counts = counts;
  P.expert_off = expert_off;
  P.rank_off = rank_off;
  P.rank_counts = rank_counts;
  P.dst_pos = dst_pos;
  P.src_idx = src_idx;
  const int nk = (E + 31) / 32;
  if (nk <= 1) return launch_small<1>(env, P);
  if (nk <= 2) return launch_small<2>(env, P);
  if (nk <= 4) return launch_small<4>(env, P);
  if (nk <= 8) return launch_small<8>(env, P);
  return launch_small<16>(env, P);
}

}  // namespace moe
