// layout_src.cu -- the per-source-rank layout: the metadata and receive
// buffers a ragged all-to-all posts, on one GPU.
//
// "GPU MoE all-to-all" (aicassindra), section "Two collectives per layer, and
// what each one moves": the per-destination counts precede the payload so
// every receiver can size its buffer; section "The message-size distribution
// is the whole story": the exchange is one logical message per (sender,
// receiver) pair.  "MoE All-to-All Dispatch and Ragged Routing", section
// "Fixed Capacity vs. Ragged Routing": rigid per-sender-expert slots.
//
// The T tokens form R source shards of Ts = ceil(T/R) consecutive tokens; the
// rows are the receive side: destination rank r, then source shard s, then
// expert e of rank r, then token order.  Segment (r, s, e) is index
// (r*R + s)*(E/R) + (e - r*(E/R)); dropless segments hold round_up(count,
// align) rows, capacity segments exactly C rows (the first C assignments of
// the pair in token order are kept).
//
// Four kernels, chained by programmatic dependent launch:
//   part count  one CTA per part (a run of TP tokens inside one shard):
//               shared-memory histogram, written whole to its workspace row
//               (no atomics to global memory, nothing to clear);
//   reduce      one CTA per chunk of 1024 segments in (rank, shard, expert)
//               order: per-segment totals from the part counts, and the
//               chunk's sums of rows and kept rows;
//   scan        one CTA per chunk: the earlier chunks' sums, then a block
//               scan of the chunk's segments (segment offsets, kept prefix);
//   place       one CTA per part (all CTAs also write the message sizes per
//               (shard, rank) and the rank slices): rank offset of each expert from the
//               earlier parts of the same shard, then each warp ranks a
//               contiguous run of assignments with __match_any_sync, warps
//               are chained in token order through per-warp counters, and
//               every assignment lands at segment start + rank (or is
//               dropped past C).  Rows without an assignment are set to -1.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kSrcThreads = 256;
constexpr int kSrcWarps = kSrcThreads / 32;
constexpr int kSegPerThread = 4;
constexpr int kChunkSeg = kSrcThreads * kSegPerThread;  // segments per reduce/scan CTA
static_assert(kChunkSeg == 1024, "layout_src_cum_words sizes the chunk sums for 1024 segments");
constexpr int kRounds = 4;  // 32-assignment rounds whose ids are loaded together

struct SrcParams {
  const int32_t* ids;
  int T, E, k, R, Er, capacity, align;
  int Ts, TP, P;
  int64_t N;
  int32_t* partc;    // [R*P][E]
  int32_t* cnt;       // [R*E] per segment, in segment order
  int32_t* keptcum;   // [R*E + 1]
  int64_t* blocksum;  // [chunks] (rows << 32) | kept per chunk of kChunkSeg segments
  WsHeader* hdr;
  int32_t* src_counts;
  int32_t* seg_off;
  int32_t* pair_counts;
  int32_t* rank_off;
  int32_t* rank_counts;
  int32_t* dst_pos;
  int32_t* src_idx;
};

// tokens [t0, t1) of part b = s*P + p
__device__ __forceinline__ void part_range(const SrcParams& P, int b, int& t0, int& t1) {
  const int s = b / P.P, p = b - (b / P.P) * P.P;
  const int64_t lo = (int64_t)s * P.Ts + (int64_t)p * P.TP;
  const int64_t hi = (int64_t)s * P.Ts + min((int64_t)(p + 1) * P.TP, (int64_t)P.Ts);
  t0 = (int)min(lo, (int64_t)P.T);
  t1 = (int)min(hi, (int64_t)P.T);
}

__global__ void __launch_bounds__(kSrcThreads) src_count_kernel(const SrcParams P) {
  extern __shared__ int32_t hist[];  // [E]
  pdl_wait();  // ids may come from the kernel launched just before
  pdl_trigger();
  for (int e = threadIdx.x; e < P.E; e += kSrcThreads) hist[e] = 0;
  __syncthreads();
  int t0, t1;
  part_range(P, blockIdx.x, t0, t1);
  for (int64_t i = (int64_t)t0 * P.k + threadIdx.x; i < (int64_t)t1 * P.k; i += kSrcThreads) {
    const int e = __ldg(P.ids + i);
    if ((unsigned)e < (unsigned)P.E)
      atomicAdd(&hist[e], 1);
    else
      report(P.hdr, MOE_ERR_DEVICE_RANGE, (int)i);
  }
  __syncthreads();
  int32_t* row = P.partc + (size_t)blockIdx.x * P.E;
  for (int e = threadIdx.x; e < P.E; e += kSrcThreads) row[e] = hist[e];
}

// (rows << 32) | kept of one segment with `cnt` assignments
__device__ __forceinline__ int64_t seg_value(const SrcParams& P, int cnt) {
  const int C = P.capacity;
  const int64_t rows = C > 0 ? C : (int64_t)((cnt + P.align - 1) / P.align) * P.align;
  const int64_t kept = (C > 0 && cnt > C) ? C : cnt;
  return (rows << 32) | kept;
}

// Sum of a 64-bit value over the CTA (kSrcThreads threads), to every thread.
__device__ int64_t sum_block64(int64_t v, int64_t* wsum) {
  constexpr int kW = kSrcThreads / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  if (lane == 0) wsum[w] = v;
  __syncthreads();
  int64_t t = 0;
#pragma unroll
  for (int q = 0; q < kW; ++q) t += wsum[q];
  __syncthreads();
  return t;
}

// Exclusive scan of a 64-bit value over the CTA (kSrcThreads threads);
// *total gets the CTA sum.
__device__ int64_t excl_scan_block64(int64_t v, int64_t* wsum, int64_t* total) {
  constexpr int kW = kSrcThreads / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  int64_t before = 0, all = 0;
#pragma unroll
  for (int q = 0; q < kW; ++q) {
    if (q < w) before += wsum[q];
    all += wsum[q];
  }
  __syncthreads();
  *total = all;
  return before + x - v;
}

// segment i = (r*R + s)*Er + el  ->  expert e and shard s
__device__ __forceinline__ void seg_coords(const SrcParams& P, int i, int& s, int& e) {
  const int per_rank = P.R * P.Er;
  const int r = i / per_rank;
  const int rem = i - r * per_rank;
  s = rem / P.Er;
  e = r * P.Er + (rem - s * P.Er);
}

// One CTA per chunk of kChunkSeg segments in (rank, shard, expert) order:
// per-segment totals from the part counts (also the caller's src_counts),
// and the chunk's sum of (rows, kept).
__global__ void __launch_bounds__(kSrcThreads) src_reduce_kernel(const SrcParams P) {
  __shared__ int64_t wsum[kSrcWarps];
  pdl_wait();  // the part counts are complete
  pdl_trigger();
  const int nseg = P.R * P.E;
  const int c0 = blockIdx.x * kChunkSeg;
  int64_t local = 0;
#pragma unroll
  for (int u = 0; u < kChunkSeg / kSrcThreads; ++u) {
    const int i = c0 + u * kSrcThreads + threadIdx.x;
    if (i < nseg) {
      int s, e;
      seg_coords(P, i, s, e);
      int cnt = 0;
      for (int p = 0; p < P.P; ++p) cnt += __ldcg(P.partc + (size_t)(s * P.P + p) * P.E + e);
      P.cnt[i] = cnt;
      P.src_counts[(size_t)s * P.E + e] = cnt;
      local += seg_value(P, cnt);
    }
  }
  const int64_t tot = sum_block64(local, wsum);
  if (threadIdx.x == 0) P.blocksum[blockIdx.x] = tot;
}

// One CTA per chunk: the sums of the earlier chunks, then an exclusive scan
// of the chunk's segments (kSegPerThread consecutive ones per thread) into
// seg_off and the kept-row prefix.
__global__ void __launch_bounds__(kSrcThreads) src_scan_kernel(const SrcParams P) {
  __shared__ int64_t wsum[kSrcWarps];
  pdl_wait();  // the totals are complete
  pdl_trigger();
  const int nseg = P.R * P.E;
  int64_t pre = 0;
  for (int c = threadIdx.x; c < (int)blockIdx.x; c += kSrcThreads) pre += __ldcg(P.blocksum + c);
  pre = sum_block64(pre, wsum);
  const int i0 = blockIdx.x * kChunkSeg + threadIdx.x * kSegPerThread;
  int64_t v[kSegPerThread];
  int64_t local = 0;
#pragma unroll
  for (int u = 0; u < kSegPerThread; ++u) {
    v[u] = (i0 + u < nseg) ? seg_value(P, __ldcg(P.cnt + i0 + u)) : 0;
    local += v[u];
  }
  int64_t total;
  int64_t run = pre + excl_scan_block64(local, wsum, &total);
#pragma unroll
  for (int u = 0; u < kSegPerThread; ++u) {
    if (i0 + u < nseg) {
      P.seg_off[i0 + u] = (int32_t)(run >> 32);
      P.keptcum[i0 + u] = (int32_t)(run & 0xffffffffll);
    }
    run += v[u];
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
    P.seg_off[nseg] = (int32_t)((pre + total) >> 32);
    P.keptcum[nseg] = (int32_t)((pre + total) & 0xffffffffll);
  }
}

__global__ void __launch_bounds__(kSrcThreads) src_place_kernel(const SrcParams P) {
  extern __shared__ int32_t sm[];
  int32_t* wc = sm;                    // [kSrcWarps][E]: warp counts, then warp bases
  int32_t* base = wc + kSrcWarps * P.E;  // [E]: rank offset from earlier parts of the shard
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int s = b / P.P, p = b - (b / P.P) * P.P;
  int t0, t1;
  part_range(P, b, t0, t1);
  const int64_t i0 = (int64_t)t0 * P.k, i1 = (int64_t)t1 * P.k;
  pdl_wait();  // the scan (and, before it, the part counts) are complete
  pdl_trigger();
  // message sizes and rank slices from the kept-row prefix (grid-stride)
  {
    const int per_rank = P.R * P.Er;
    const int nthr = gridDim.x * kSrcThreads;
    const int tid = b * kSrcThreads + threadIdx.x;
    for (int q = tid; q < P.R * P.R; q += nthr) {  // q = s*R + r
      const int sq = q / P.R, r = q - (q / P.R) * P.R;
      const int lo = (r * P.R + sq) * P.Er;
      P.pair_counts[q] = __ldcg(P.keptcum + lo + P.Er) - __ldcg(P.keptcum + lo);
    }
    for (int r = tid; r <= P.R; r += nthr) {
      P.rank_off[r] = __ldcg(P.seg_off + (size_t)r * per_rank);
      if (r < P.R)
        P.rank_counts[r] = __ldcg(P.keptcum + (size_t)(r + 1) * per_rank) -
                           __ldcg(P.keptcum + (size_t)r * per_rank);
    }
  }
  for (int x = threadIdx.x; x < kSrcWarps * P.E; x += kSrcThreads) wc[x] = 0;
  for (int e = threadIdx.x; e < P.E; e += kSrcThreads) {
    int pre = 0;
    for (int q = 0; q < p; ++q) pre += __ldcg(P.partc + (size_t)(s * P.P + q) * P.E + e);
    base[e] = pre;
  }
  __syncthreads();

  // each warp: a contiguous run of the part's assignments (whole 32-lane rounds)
  const int64_t chunk = (((i1 - i0) + kSrcWarps - 1) / kSrcWarps + 31) / 32 * 32;
  const int64_t s0 = min(i1, i0 + (int64_t)w * chunk);
  const int64_t s1 = min(i1, s0 + chunk);
  int32_t* my = wc + w * P.E;
  // rank of every assignment inside the warp's run; `emit` sees (i, e, rank)
  // with rank -1 for an invalid id
  auto run = [&](auto&& emit) {
    for (int64_t r0 = s0; r0 < s1; r0 += 32 * kRounds) {
      int ev[kRounds];
#pragma unroll
      for (int u = 0; u < kRounds; ++u) {  // loads of kRounds rounds in flight
        const int64_t i = r0 + 32 * u + lane;
        ev[u] = i < s1 ? __ldg(P.ids + i) : -1;
      }
#pragma unroll
      for (int u = 0; u < kRounds; ++u) {
        const int64_t i = r0 + 32 * u + lane;
        if (r0 + 32 * u >= s1) break;  // warp-uniform
        const int e = ev[u];
        const bool ok = i < s1 && (unsigned)e < (unsigned)P.E;
        const unsigned active = __ballot_sync(kFull, ok);
        int v = -1;
        if (ok) {
          const unsigned peers = __match_any_sync(active, e);
          v = my[e] + __popc(peers & lanemask_lt());
          __syncwarp(active);
          if (lane == __ffs(peers) - 1) my[e] = v + __popc(peers);
        }
        __syncwarp();
        if (i < s1) emit(i, e, v);
      }
    }
  };
  run([](int64_t, int, int) {});
  __syncthreads();
  for (int e = threadIdx.x; e < P.E; e += kSrcThreads) {  // warp counts -> bases
    int acc = base[e];
    for (int q = 0; q < kSrcWarps; ++q) {
      const int c = wc[q * P.E + e];
      wc[q * P.E + e] = acc;
      acc += c;
    }
  }
  __syncthreads();
  const int C = P.capacity;
  run([&](int64_t i, int e, int rank) {
    int64_t dst = -1;
    if (rank >= 0 && (C == 0 || rank < C)) {
      const int r = e / P.Er;
      const int seg = (r * P.R + s) * P.Er + (e - r * P.Er);
      dst = (int64_t)__ldg(P.seg_off + seg) + rank;
      if (dst >= P.N) {  // in range by construction; guards corrupted counts
        report(P.hdr, MOE_ERR_DEVICE_RANGE, (int)(dst > INT32_MAX ? INT32_MAX : dst));
        dst = -1;
      }
    }
    P.dst_pos[i] = (int32_t)dst;
    if (dst >= 0) P.src_idx[dst] = (int32_t)i;
  });

  // rows that hold no assignment: alignment padding, unused capacity slots
  if (C > 0 || P.align > 1) {
    const int nseg = P.R * P.E;
    const int64_t per = (P.N + gridDim.x - 1) / gridDim.x;
    const int64_t r0 = (int64_t)b * per, r1 = min(P.N, r0 + per);
    const int used = __ldg(P.seg_off + nseg);
    for (int64_t row = r0 + threadIdx.x; row < r1; row += kSrcThreads) {
      bool pad = true;
      if (row < used) {
        int lo = 0, hi = nseg - 1;  // last segment starting at or before row
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (__ldg(P.seg_off + mid) <= row)
            lo = mid;
          else
            hi = mid - 1;
        }
        const int per_rank = P.R * P.Er;
        const int r = lo / per_rank, rem = lo - (lo / per_rank) * per_rank;
        const int sh = rem / P.Er, e = r * P.Er + (rem - (rem / P.Er) * P.Er);
        const int cnt = __ldg(P.src_counts + (size_t)sh * P.E + e);
        const int kept = (C > 0 && cnt > C) ? C : cnt;
        pad = (row - __ldg(P.seg_off + lo)) >= kept;
      }
      if (pad) P.src_idx[row] = -1;
    }
  }
}

}  // namespace

cudaError_t launch_layout_src(const LaunchEnv& env, const int32_t* ids, int T, int E, int k, int R,
                              int capacity, int align, int64_t N, int32_t* partc,
                              int32_t* scratch, WsHeader* hdr, int32_t* src_counts,
                              int32_t* seg_off, int32_t* pair_counts, int32_t* rank_off,
                              int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx) {
  const SrcGeom g = layout_src_geom(T, R);
  SrcParams P;
  P.ids = ids;
  P.T = T;
  P.E = E;
  P.k = k;
  P.R = R;
  P.Er = E / R;
  P.capacity = capacity;
  P.align = align;
  P.Ts = g.Ts;
  P.TP = g.TP;
  P.P = g.P;
  P.N = N;
  P.partc = partc;
  P.cnt = scratch;
  P.keptcum = scratch + ((size_t)R * E + 3) / 4 * 4;
  P.blocksum = reinterpret_cast<int64_t*>(P.keptcum + ((size_t)R * E + 1 + 3) / 4 * 4);
  P.hdr = hdr;
  P.src_counts = src_counts;
  P.seg_off = seg_off;
  P.pair_counts = pair_counts;
  P.rank_off = rank_off;
  P.rank_counts = rank_counts;
  P.dst_pos = dst_pos;
  P.src_idx = src_idx;
  const unsigned parts = (unsigned)(R * g.P);
  const size_t count_smem = (size_t)E * sizeof(int32_t);
  const size_t place_smem = (size_t)(kSrcWarps + 1) * E * sizeof(int32_t);
  int per_sm = 1;
  cudaError_t err =
      blocks_per_sm(reinterpret_cast<const void*>(src_count_kernel), kSrcThreads, count_smem, &per_sm);
  if (err != cudaSuccess) return err;
  err = blocks_per_sm(reinterpret_cast<const void*>(src_place_kernel), kSrcThreads, place_smem,
                      &per_sm);
  if (err != cudaSuccess) return err;
  err = launch_pdl(env, src_count_kernel, dim3(parts), dim3(kSrcThreads), count_smem, P);
  if (err != cudaSuccess) return err;
  const unsigned chunks = (unsigned)(((int64_t)R * E + kChunkSeg - 1) / kChunkSeg);
  err = launch_pdl(env, src_reduce_kernel, dim3(chunks), dim3(kSrcThreads), 0, P);
  if (err != cudaSuccess) return err;
  err = launch_pdl(env, src_scan_kernel, dim3(chunks), dim3(kSrcThreads), 0, P);
  if (err != cudaSuccess) return err;
  return launch_pdl(env, src_place_kernel, dim3(parts), dim3(kSrcThreads), place_smem, P);
}

}  // namespace moe
