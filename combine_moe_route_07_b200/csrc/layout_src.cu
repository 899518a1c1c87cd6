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
// Three kernels, chained by programmatic dependent launch:
//   part count  one CTA per part (a run of TP tokens inside one shard):
//               shared-memory histogram, written whole to its workspace row
//               (no atomics to global memory, nothing to clear);
//   scan        one CTA: per-(shard, expert) totals, segment sizes and kept
//               rows in (rank, shard, expert) order, one block scan per
//               4096 segments with a running carry; message sizes per
//               (shard, rank) and rank slices from the kept-row prefix;
//   place       one CTA per part: rank offset of each expert from the
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
constexpr int kScanThreads = 1024;
constexpr int kScanPer = 4;  // segments per thread per scan chunk

struct SrcParams {
  const int32_t* ids;
  int T, E, k, R, Er, capacity, align;
  int Ts, TP, P;
  int64_t N;
  int32_t* partc;    // [R*P][E]
  int32_t* keptcum;  // [R*E + 1]
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

// Inclusive scan of a 64-bit value across the CTA (kScanThreads threads);
// returns the inclusive prefix, and the CTA total in *total.
__device__ int64_t scan_block64(int64_t v, int64_t* wsum, int64_t* total) {
  constexpr int kW = kScanThreads / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  if (w == 0) {
    int64_t s = lane < kW ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(kFull, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kW) wsum[lane] = s;
  }
  __syncthreads();
  const int64_t r = x + (w > 0 ? wsum[w - 1] : 0);
  *total = wsum[kW - 1];
  __syncthreads();  // wsum is reused by the next call
  return r;
}

__global__ void __launch_bounds__(kScanThreads) src_scan_kernel(const SrcParams P) {
  __shared__ int64_t wsum[kScanThreads / 32];
  pdl_wait();  // the part counts are complete
  pdl_trigger();
  const int nseg = P.R * P.E;
  const int C = P.capacity;
  const int per_rank = P.R * P.Er;  // segments of one destination rank (= E)
  int64_t carry = 0;                // (rows << 32) | kept, summed so far
  for (int c0 = 0; c0 < nseg; c0 += kScanThreads * kScanPer) {
    int64_t v[kScanPer];
    int64_t local = 0;
#pragma unroll
    for (int u = 0; u < kScanPer; ++u) {
      const int i = c0 + threadIdx.x * kScanPer + u;
      v[u] = 0;
      if (i < nseg) {
        const int r = i / per_rank;
        const int rem = i - r * per_rank;
        const int s = rem / P.Er;
        const int e = r * P.Er + (rem - s * P.Er);
        int cnt = 0;
        for (int p = 0; p < P.P; ++p) cnt += __ldcg(P.partc + (size_t)(s * P.P + p) * P.E + e);
        P.src_counts[(size_t)s * P.E + e] = cnt;
        const int64_t rows = C > 0 ? C : (int64_t)((cnt + P.align - 1) / P.align) * P.align;
        const int64_t kept = (C > 0 && cnt > C) ? C : cnt;
        v[u] = (rows << 32) | kept;
      }
      local += v[u];
    }
    int64_t total;
    const int64_t incl = scan_block64(local, wsum, &total);
    int64_t run = carry + incl - local;
#pragma unroll
    for (int u = 0; u < kScanPer; ++u) {
      const int i = c0 + threadIdx.x * kScanPer + u;
      if (i < nseg) {
        P.seg_off[i] = (int32_t)(run >> 32);
        P.keptcum[i] = (int32_t)(run & 0xffffffffll);
      }
      run += v[u];
    }
    carry += total;
  }
  if (threadIdx.x == 0) {
    P.seg_off[nseg] = (int32_t)(carry >> 32);
    P.keptcum[nseg] = (int32_t)(carry & 0xffffffffll);
  }
  __syncthreads();  // this CTA's global writes above are visible below
  for (int q = threadIdx.x; q < P.R * P.R; q += kScanThreads) {  // q = s*R + r
    const int s = q / P.R, r = q - (q / P.R) * P.R;
    const int lo = (r * P.R + s) * P.Er;
    P.pair_counts[q] = __ldcg(P.keptcum + lo + P.Er) - __ldcg(P.keptcum + lo);
  }
  for (int r = threadIdx.x; r <= P.R; r += kScanThreads) {
    P.rank_off[r] = __ldcg(P.seg_off + (size_t)r * per_rank);
    if (r < P.R)
      P.rank_counts[r] =
          __ldcg(P.keptcum + (size_t)(r + 1) * per_rank) - __ldcg(P.keptcum + (size_t)r * per_rank);
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
    for (int64_t r0 = s0; r0 < s1; r0 += 32) {
      const int64_t i = r0 + lane;
      const int e = i < s1 ? __ldg(P.ids + i) : -1;
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
                              int32_t* keptcum, WsHeader* hdr, int32_t* src_counts,
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
  P.keptcum = keptcum;
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
  err = launch_pdl(env, src_scan_kernel, dim3(1), dim3(kScanThreads), 0, P);
  if (err != cudaSuccess) return err;
  return launch_pdl(env, src_place_kernel, dim3(parts), dim3(kSrcThreads), place_smem, P);
}

}  // namespace moe
