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
// Two kernels, chained by programmatic dependent launch (the kernel boundary
// is the only grid-wide synchronisation; nothing spins):
//
//  count  CTAs over groups of 16 tokens: shared-memory histogram of the
//         group's expert ids, added into the row of the tile (TT consecutive
//         tokens, about 128 tiles) the group lies in.  The fused route path
//         does this inside the route kernel instead.
//  place  one CTA per tile.  It sums every tile row at once (16-byte loads,
//         one warp per row stride), so it knows each expert's total and its
//         count in earlier tiles; a shared-memory scan over experts gives the
//         expert offsets (segments rounded to `align`, or C rows each).  Then
//         one pass over the tile's assignments, each warp over a contiguous
//         run: __match_any_sync groups equal ids and the group leader advances
//         the warp's counter, giving each assignment its rank inside the run.
//         Token-order rank in the expert = earlier tiles + earlier warps of
//         this tile + rank in the run.  CTA 0 writes counts and offsets.
//
// The tile counts live in one of two tables, alternating per call: a place
// pass reads the table its count pass filled and clears the other one (the
// rows the previous call left), so no clearing sits on the critical path.
// Integer adds make every result independent of the order the CTAs run in.
#include "block_scan.cuh"
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kCountThreads = 256;
constexpr int kPlaceThreads = 512;
constexpr int kUnroll = 4;
constexpr int kMaxStaged = 8192;  // assignments per tile kept in smem across the passes
constexpr int kRowsInFlight = 8;  // tile rows each warp loads before adding

__global__ void __launch_bounds__(kCountThreads)
    count_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int TT,
                 uint32_t* __restrict__ tables, size_t half_words, WsHeader* hdr) {
  extern __shared__ int32_t hist[];  // [E]
  pdl_wait();  // ids (and the tables) may come from the kernel launched before
  pdl_trigger();
  const uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(&hdr->epoch);
  uint32_t* tab = tables + (size_t)(epoch & 1u) * half_words;
  for (int e = threadIdx.x; e < E; e += kCountThreads) hist[e] = 0;
  __syncthreads();
  for (int g0 = blockIdx.x * kLayoutTileQuantum; g0 < T; g0 += gridDim.x * kLayoutTileQuantum) {
    const int64_t i0 = (int64_t)g0 * k;
    const int64_t i1 = (int64_t)min(T, g0 + kLayoutTileQuantum) * k;
    for (int64_t i = i0 + threadIdx.x; i < i1; i += kCountThreads) {
      const int e = __ldg(ids + i);
      if ((unsigned)e < (unsigned)E)
        atomicAdd(&hist[e], 1);
      else
        report(hdr, MOE_ERR_DEVICE_RANGE, (int)i);
    }
    __syncthreads();
    uint32_t* row = tab + (size_t)(g0 / TT) * E;  // the group lies in one tile
    for (int e = threadIdx.x; e < E; e += kCountThreads) {
      const int c = hist[e];
      if (c != 0) {
        atomicAdd(row + e, (uint32_t)c);
        hist[e] = 0;
      }
    }
    __syncthreads();
  }
}

struct PlaceParams {
  const int32_t* ids;
  int T, k, E, R, capacity, align, G, TT;
  int home;             // slices in rank order home+1, ..., home (mod R); R-1: natural order
  int32_t* tile_expert;  // [N/align] expert of each align-row tile, or nullptr
  int staged;
  int64_t N;
  uint32_t* tables;
  size_t half_words;
  WsHeader* hdr;
  int32_t* counts;
  int32_t* expert_off;
  int32_t* rank_off;
  int32_t* rank_counts;
  int32_t* dst_pos;
  int32_t* src_idx;
};

constexpr size_t place_smem_words(int E, int staged_entries) {
  return (size_t)(kPlaceThreads / 32) * E + 5 * (size_t)E + 2 + 2 * (size_t)staged_entries;
}

// Expert at position q of the slice order (ranks home+1, home+2, ... mod R).
__device__ __forceinline__ int slice_expert(int q, int home, int R, int Er) {
  return ((home + 1 + q / Er) % R) * Er + q % Er;
}

__global__ void __launch_bounds__(kPlaceThreads) place_kernel(const PlaceParams P) {
  constexpr int kW = kPlaceThreads / 32;
  extern __shared__ int32_t smem[];
  const int E = P.E, k = P.k, C = P.capacity;
  int32_t* wh = smem;             // [kW][E] per-warp counts, then tile-local warp bases
  int32_t* pre = wh + kW * E;     // [E] count in earlier tiles
  int32_t* tot = pre + E;         // [E] total count
  int32_t* off = tot + E;         // [E+1] expert offsets
  int32_t* kept = off + E + 1;    // [E] rows kept per expert
  int32_t* offq = kept + E;       // [E+1] segment starts in slice order (increasing)
  int32_t* sid = offq + E + 1;    // [TT*k] staged expert ids
  int32_t* srk = sid + P.TT * k;  // [TT*k] staged ranks inside the warp's run
  __shared__ int32_t s_wtot[kW];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vb = blockIdx.x;
  const int t0 = min(P.T, vb * P.TT);
  const int t1 = min(P.T, t0 + P.TT);
  const int64_t i0 = (int64_t)t0 * k, i1 = (int64_t)t1 * k;

  pdl_wait();  // the count pass has finished
  pdl_trigger();
  // epoch, done, words_used[0..1] in one load
  const uint4 hv = __ldcg(reinterpret_cast<const uint4*>(&P.hdr->epoch));
  const uint32_t epoch = hv.x;
  const uint32_t cur_b = epoch & 1u, oth_b = cur_b ^ 1u;
  const uint32_t* cur = P.tables + (size_t)cur_b * P.half_words;
  uint32_t* oth = P.tables + (size_t)oth_b * P.half_words;
  const uint32_t oth_used = oth_b ? hv.w : hv.z;
  for (int i = threadIdx.x; i < kW * E; i += kPlaceThreads) wh[i] = 0;
  for (int e = threadIdx.x; e < E; e += kPlaceThreads) {
    pre[e] = 0;
    tot[e] = 0;
  }
  // this warp's contiguous run of the tile's assignments; its first ids are
  // fetched now so their latency overlaps the table reads below
  const int64_t chunk = (((i1 - i0) + kW - 1) / kW + 31) / 32 * 32;
  const int64_t s0 = min(i1, i0 + (int64_t)w * chunk);
  const int64_t s1 = min(i1, s0 + chunk);
  int ev0[kUnroll];
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int64_t i = s0 + 32 * u + lane;
    ev0[u] = (i < s1) ? __ldg(P.ids + i) : -1;
  }
  __syncthreads();

  // 1. every tile row: totals and the count in earlier tiles
  if ((E & 3) == 0) {
    for (int eb = 4 * lane; eb < E; eb += 128) {
      uint4 at = make_uint4(0, 0, 0, 0), ap = make_uint4(0, 0, 0, 0);
      for (int p0 = w; p0 < P.G; p0 += kW * kRowsInFlight) {
        uint4 v[kRowsInFlight];
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
          const int p = p0 + r * kW;
          v[r] = (p < P.G) ? __ldcg(reinterpret_cast<const uint4*>(cur + (size_t)p * E + eb))
                           : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
          at.x += v[r].x;
          at.y += v[r].y;
          at.z += v[r].z;
          at.w += v[r].w;
          if (p0 + r * kW < vb) {
            ap.x += v[r].x;
            ap.y += v[r].y;
            ap.z += v[r].z;
            ap.w += v[r].w;
          }
        }
      }
      atomicAdd(&tot[eb + 0], (int)at.x);
      atomicAdd(&tot[eb + 1], (int)at.y);
      atomicAdd(&tot[eb + 2], (int)at.z);
      atomicAdd(&tot[eb + 3], (int)at.w);
      atomicAdd(&pre[eb + 0], (int)ap.x);
      atomicAdd(&pre[eb + 1], (int)ap.y);
      atomicAdd(&pre[eb + 2], (int)ap.z);
      atomicAdd(&pre[eb + 3], (int)ap.w);
    }
  } else {
    for (int e = lane; e < E; e += 32) {
      int at = 0, ap = 0;
      for (int p = w; p < P.G; p += kW) {
        const int v = (int)__ldcg(cur + (size_t)p * E + e);
        at += v;
        if (p < vb) ap += v;
      }
      atomicAdd(&tot[e], at);
      atomicAdd(&pre[e], ap);
    }
  }
  __syncthreads();

  // 2. expert offsets (every CTA computes the same scan, in slice order);
  //    CTA 0 publishes them
  const int Er = E / P.R;
  for (int e = threadIdx.x; e < E; e += kPlaceThreads) {
    const int c = tot[e];
    kept[e] = (C > 0 && c > C) ? C : c;
  }
  for (int q = threadIdx.x; q < E; q += kPlaceThreads) {
    const int c = tot[slice_expert(q, P.home, P.R, Er)];
    offq[q] = C > 0 ? C : ((c + P.align - 1) / P.align) * P.align;
  }
  __syncthreads();
  const int used = block_exclusive_scan<kPlaceThreads>(offq, E, s_wtot);
  for (int q = threadIdx.x; q < E; q += kPlaceThreads) off[slice_expert(q, P.home, P.R, Er)] = offq[q];
  if (threadIdx.x == 0) {
    off[E] = used;
    offq[E] = used;
  }
  __syncthreads();
  if (vb == 0) {
    for (int e = threadIdx.x; e < E; e += kPlaceThreads) {
      P.counts[e] = tot[e];
      P.expert_off[e] = off[e];
    }
    for (int r = w; r < P.R; r += kW) {  // one warp per rank: rows kept
      int s = 0;
      for (int e = r * Er + lane; e < (r + 1) * Er; e += 32) s += kept[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
      if (lane == 0) {
        P.rank_counts[r] = s;
        P.rank_off[r] = off[r * Er];
      }
    }
    if (threadIdx.x == 0) {
      P.expert_off[E] = used;
      P.rank_off[P.R] = used;
    }
  }

  // 3. this tile's assignments: per-warp counts and each one's rank in its run
  int32_t* my = wh + w * E;
  auto run_ranks = [&](auto&& emit, bool first_prefetched) {
    for (int64_t base = s0; base < s1; base += 32 * kUnroll) {
      int ev[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + 32 * u + lane;
        ev[u] = (first_prefetched && base == s0) ? ev0[u] : ((i < s1) ? __ldg(P.ids + i) : -1);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + 32 * u + lane;
        if (base + 32 * u < s1) {
          const int e = ev[u];
          const bool ok = (i < s1) && (unsigned)e < (unsigned)E;
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
    }
  };
  if (P.staged)
    run_ranks(
        [&](int64_t i, int e, int v) {
          sid[i - i0] = e;
          srk[i - i0] = v;
        },
        true);
  else
    run_ranks([](int64_t, int, int) {}, true);
  __syncthreads();
  // per-warp counts -> tile-local bases (warps in token order)
  for (int e = threadIdx.x; e < E; e += kPlaceThreads) {
    int run = pre[e];
    for (int q = 0; q < kW; ++q) {
      const int c = wh[q * E + e];
      wh[q * E + e] = run;
      run += c;
    }
  }
  __syncthreads();

  // 4. place each assignment at its row
  auto place = [&](int64_t i, int e, int rank) {
    int64_t dst = -1;
    if (rank >= 0)
      dst = (C > 0 && rank >= C) ? -1 : (int64_t)off[e] + rank;
    if (dst >= P.N) {  // in range by construction; guards a corrupted tile table
      report(P.hdr, MOE_ERR_DEVICE_RANGE, (int)(dst > INT32_MAX ? INT32_MAX : dst));
      dst = -1;
    }
    P.dst_pos[i] = (int32_t)dst;
    if (dst >= 0) P.src_idx[dst] = (int32_t)i;
  };
  if (P.staged) {
    for (int64_t r = threadIdx.x; r < i1 - i0; r += kPlaceThreads) {
      const int e = sid[r];
      const int v = srk[r];
      const int q = (int)(r / chunk);  // the warp whose run holds r
      place(i0 + r, e, v < 0 ? -1 : wh[q * E + e] + v);
    }
  } else {
    run_ranks([&](int64_t i, int e, int v) { place(i, e, v); }, true);  // my[] starts at the bases
  }

  // 5. rows that hold no assignment (alignment padding, unused capacity
  //    slots), and the tile map; segments are searched in slice order
  auto segment_of = [&](int64_t row) {  // last q with offq[q] <= row (row < used)
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (offq[mid] <= row)
        lo = mid;
      else
        hi = mid - 1;
    }
    return lo;
  };
  if (C > 0 || P.align > 1) {
    const int64_t per = (P.N + P.G - 1) / P.G;
    const int64_t r0 = (int64_t)vb * per;
    const int64_t r1 = min(P.N, r0 + per);
    for (int64_t p = r0 + threadIdx.x; p < r1; p += kPlaceThreads) {
      bool pad = true;
      if (p < offq[E]) {
        const int q = segment_of(p);
        pad = (p - offq[q]) >= kept[slice_expert(q, P.home, P.R, Er)];
      }
      if (pad) P.src_idx[p] = -1;
    }
  }
  if (P.tile_expert != nullptr) {
    const int64_t ntiles = P.N / P.align;
    const int64_t per = (ntiles + P.G - 1) / P.G;
    const int64_t a0 = (int64_t)vb * per;
    const int64_t a1 = min(ntiles, a0 + per);
    for (int64_t i = a0 + threadIdx.x; i < a1; i += kPlaceThreads) {
      const int64_t row = i * P.align;
      P.tile_expert[i] =
          row < offq[E] ? slice_expert(segment_of(row), P.home, P.R, Er) : -1;
    }
  }

  // 6. clear what the previous call left in the other table; the last CTA to
  //    finish flips the tables for the next call
  for (size_t x = (size_t)vb * kPlaceThreads + threadIdx.x; x < oth_used;
       x += (size_t)P.G * kPlaceThreads)
    oth[x] = 0u;
  // (everything here is read only by the next call, after this kernel has
  // completed, so the counter needs no fence)
  __syncthreads();
  if (threadIdx.x == 0) {
    if (atomicAdd(&P.hdr->done, 1u) == (uint32_t)P.G - 1u) {
      P.hdr->words_used[cur_b] = (uint32_t)((size_t)P.G * E);
      P.hdr->words_used[oth_b] = 0u;
      P.hdr->done = 0u;
      P.hdr->epoch = epoch + 1u;
    }
  }
}

}  // namespace

cudaError_t launch_layout(const LaunchEnv& env, const int32_t* ids, int T, int E, int k, int R,
                          int capacity, int align, int64_t N, uint32_t* tables,
                          size_t half_words, WsHeader* hdr, int32_t* counts, int32_t* expert_off,
                          int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                          int32_t* src_idx, bool count_ids, int home, int32_t* tile_expert) {
  const TileGeom geom = layout_tiles(T);
  cudaError_t err;
  if (count_ids && T > 0) {
    const size_t smem = (size_t)E * sizeof(int32_t);
    int per_sm = 1;
    err = blocks_per_sm(reinterpret_cast<const void*>(count_kernel), kCountThreads, smem, &per_sm);
    if (err != cudaSuccess) return err;
    int64_t blocks = ((int64_t)T + kLayoutTileQuantum - 1) / kLayoutTileQuantum;
    const int64_t cap = (int64_t)per_sm * env.num_sms;
    if (blocks > cap) blocks = cap;
    err = launch_pdl(env, count_kernel, dim3((unsigned)blocks), dim3(kCountThreads), smem, ids, T,
                     k, E, geom.TT, tables, half_words, hdr);
    if (err != cudaSuccess) return err;
  }
  PlaceParams P{};
  P.ids = ids;
  P.T = T;
  P.k = k;
  P.E = E;
  P.R = R;
  P.capacity = capacity;
  P.align = align;
  P.home = (home >= 0 && home < R) ? home : R - 1;
  P.tile_expert = tile_expert;
  P.G = geom.G;
  P.TT = geom.TT;
  P.N = N;
  P.tables = tables;
  P.half_words = half_words;
  P.hdr = hdr;
  P.counts = counts;
  P.expert_off = expert_off;
  P.rank_off = rank_off;
  P.rank_counts = rank_counts;
  P.dst_pos = dst_pos;
  P.src_idx = src_idx;
  const int64_t entries = (int64_t)geom.TT * k;
  P.staged = entries <= kMaxStaged ? 1 : 0;
  const size_t smem = place_smem_words(E, P.staged ? (int)entries : 0) * sizeof(int32_t);
  int per_sm = 1;  // (raises the kernel's dynamic shared-memory limit to smem)
  err = blocks_per_sm(reinterpret_cast<const void*>(place_kernel), kPlaceThreads, smem, &per_sm);
  if (err != cudaSuccess) return err;
  return launch_pdl(env, place_kernel, dim3((unsigned)geom.G), dim3(kPlaceThreads), smem, P);
}

}  // namespace moe
