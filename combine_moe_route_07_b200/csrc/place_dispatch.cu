// place_dispatch.cu -- steps 3 and 4 in one kernel behind the route kernel:
// each CTA places a contiguous range of tokens and streams their rows.
//
// "GPU MoE all-to-all" (aicassindra), section "Bucketing: cut the message
// count, not the byte count": the permutation is fused into the kernel that
// stages the rows; section "Two collectives per layer": the per-destination
// counts (here the route kernel's per-tile histograms) come first.
//
// The route kernel leaves one row of expert counts per layout tile (TT
// consecutive tokens) in the workspace table.  CTA b of this kernel owns the
// tokens [a0, a1) (a balanced contiguous range, not aligned to tiles) and:
//   0. starts bulk loads of its first x rows into its pipelines' rings (x is
//      complete: this kernel runs right behind the library's route kernel);
//   1. reads every tile row (16-byte loads through L2): each expert's total,
//      and its count in the tiles before a0's tile; adds the assignments of
//      the tokens of that tile before a0 (read from ids): the count of every
//      expert in the tokens before a0;
//   2. scans the expert offsets (dropless, segments rounded to `align`),
//      ranks its own assignments in token order (__match_any_sync per warp
//      run) and writes dst_pos and src_idx; CTA 0 writes counts and offsets,
//      every CTA a share of the padding rows and of the clearing of the table
//      the previous call filled; the last CTA to finish flips the tables;
//   3. streams its rows: kPdPipes warps, each a ring of shared-memory stages,
//      one bulk load of a row and k bulk stores of it.
// Against a place kernel followed by the dispatch kernel, the placement runs
// in the CTAs that store the rows, under their x loads, with one kernel
// boundary fewer: Prefill 120.5 -> 120.1 us a step.  Every wait is bounded.
// The results are the same bits as the place and dispatch kernels.
#include <cuda_runtime.h>

#include "block_scan.cuh"
#include "bulk.cuh"
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kPdThreads = 512;
constexpr int kPdWarps = kPdThreads / 32;
constexpr int kPdPipes = 4;       // warps that stream the rows
constexpr int kPdMaxStages = 8;   // ring stages per pipeline
constexpr int kPdMinStages = 2;
constexpr int kPdRowsInFlight = 8;
constexpr int kPdMaxAssign = 512;   // assignments in a CTA's range
constexpr size_t kPdSmemBudget = 200u * 1024u;
constexpr uint64_t kPdTimeoutNs = 1000000000ull;

struct PdParams {
  const int32_t* ids;
  const char* x;
  int T, E, k, R, align;
  int G, TT;       // the route kernel's tiles: G rows of TT tokens
  int TB;          // tokens per CTA
  int stages;      // ring stages per pipeline
  uint32_t row;    // bytes per row
  int evict_first;
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
  char* out;
};

size_t pd_int_words(int E, int TB, int k) {
  return (size_t)kPdWarps * E + 4 * (size_t)E + 1 + 2 * (size_t)TB * k;
}

__global__ void __launch_bounds__(kPdThreads, 1) place_dispatch_kernel(const PdParams P) {
  // dynamic: ring [kPdPipes][stages][row] bytes, then wh[kPdWarps][E]
  // (per-warp counts, then bases), pre[E], tot[E], off[E+1], kept[E],
  // sid[TB*k] (ids), sdst[TB*k] (rank in the warp's run, then the row)
  extern __shared__ __align__(128) unsigned char dyn[];
  __shared__ uint64_t bars[kPdPipes][kPdMaxStages];
  __shared__ int32_t s_wtot[kPdWarps];
  const int E = P.E, k = P.k, T = P.T;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a0 = min(T, (int)blockIdx.x * P.TB), a1 = min(T, a0 + P.TB);
  const int nt = a1 - a0, n = nt * k;
  const uint32_t row = P.row;
  const int stages = P.stages;
  int32_t* wh = reinterpret_cast<int32_t*>(dyn + (size_t)kPdPipes * stages * row);
  int32_t* pre = wh + kPdWarps * E;
  int32_t* tot = pre + E;
  int32_t* off = tot + E;
  int32_t* kept = off + E + 1;
  int32_t* sid = kept + E;
  int32_t* sdst = sid + P.TB * k;

  // 0. pipeline w streams the tokens a0 + w + kPdPipes*j through its stages;
  //    its first stages-1 rows are requested now
  unsigned char* ring = dyn + (size_t)w * stages * row;
  const int cnt = w < kPdPipes && w < nt ? (nt - 1 - w) / kPdPipes + 1 : 0;
  auto issue_load = [&](int j) {
    const int s = j % stages;
    mbar_arrive_expect_tx(&bars[w][s], row);
    bulk_load(ring + (size_t)s * row, P.x + (size_t)(a0 + w + kPdPipes * j) * row, row,
              &bars[w][s]);
  };
  int issued = 0;
  if (w < kPdPipes && lane == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&bars[w][s], 1);
    mbar_fence_init();
    for (; issued < cnt && issued < stages - 1; ++issued) issue_load(issued);
  }
  pdl_wait();  // the route kernel's tile table and ids are complete
  pdl_trigger();

  // 1. every tile row: totals, and the count in the tiles before a0's tile
  const uint4 hv = __ldcg(reinterpret_cast<const uint4*>(&P.hdr->epoch));
  const uint32_t epoch = hv.x;
  const uint32_t cur_b = epoch & 1u, oth_b = cur_b ^ 1u;
  const uint32_t* cur = P.tables + (size_t)cur_b * P.half_words;
  uint32_t* oth = P.tables + (size_t)oth_b * P.half_words;
  const uint32_t oth_used = oth_b ? hv.w : hv.z;
  for (int i = threadIdx.x; i < kPdWarps * E; i += kPdThreads) wh[i] = 0;
  for (int e = threadIdx.x; e < E; e += kPdThreads) {
    pre[e] = 0;
    tot[e] = 0;
  }
  __syncthreads();
  const int tile0 = a0 / P.TT;  // a0's tile; its tokens before a0 are counted from ids
  if ((E & 3) == 0) {
    for (int eb = 4 * lane; eb < E; eb += 128) {
      uint4 at = make_uint4(0, 0, 0, 0), ap = make_uint4(0, 0, 0, 0);
      for (int p0 = w; p0 < P.G; p0 += kPdWarps * kPdRowsInFlight) {
        uint4 v[kPdRowsInFlight];
#pragma unroll
        for (int r = 0; r < kPdRowsInFlight; ++r) {
          const int p = p0 + r * kPdWarps;
          v[r] = (p < P.G) ? __ldcg(reinterpret_cast<const uint4*>(cur + (size_t)p * E + eb))
                           : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < kPdRowsInFlight; ++r) {
          at.x += v[r].x;
          at.y += v[r].y;
          at.z += v[r].z;
          at.w += v[r].w;
          if (p0 + r * kPdWarps < tile0) {
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
      for (int p = w; p < P.G; p += kPdWarps) {
        const int v = (int)__ldcg(cur + (size_t)p * E + e);
        at += v;
        if (p < tile0) ap += v;
      }
      atomicAdd(&tot[e], at);
      atomicAdd(&pre[e], ap);
    }
  }
  //    the assignments of a0's tile before a0, and this range's ids
  for (int64_t i = (int64_t)tile0 * P.TT * k + threadIdx.x; i < (int64_t)a0 * k;
       i += kPdThreads) {
    const int e = __ldg(P.ids + i);
    if ((unsigned)e < (unsigned)E) atomicAdd(&pre[e], 1);
  }
  for (int i = threadIdx.x; i < n; i += kPdThreads) {
    const int e = __ldg(P.ids + (size_t)a0 * k + i);
    if ((unsigned)e >= (unsigned)E) report(P.hdr, MOE_ERR_DEVICE_RANGE, a0 * k + i);
    sid[i] = e;
  }
  __syncthreads();

  // 2. expert offsets (every CTA the same scan); CTA 0 publishes them
  for (int e = threadIdx.x; e < E; e += kPdThreads) {
    const int c = tot[e];
    kept[e] = c;
    off[e] = ((c + P.align - 1) / P.align) * P.align;
  }
  __syncthreads();
  const int used = block_exclusive_scan<kPdThreads>(off, E, s_wtot);  // (synchronises the CTA)
  if (threadIdx.x == 0) off[E] = used;
  __syncthreads();
  if (blockIdx.x == 0) {
    const int Er = E / P.R;
    for (int e = threadIdx.x; e < E; e += kPdThreads) P.counts[e] = tot[e];
    for (int e = threadIdx.x; e <= E; e += kPdThreads) P.expert_off[e] = off[e];
    for (int r = w; r < P.R; r += kPdWarps) {  // one warp per rank: rows kept
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
  //    token-order ranks of this range's assignments: warp w a contiguous run
  const int chunk = ((n + kPdWarps - 1) / kPdWarps + 31) / 32 * 32;
  const int s0 = min(n, w * chunk), s1 = min(n, s0 + chunk);
  int32_t* my = wh + w * E;
  for (int r0 = s0; r0 < s1; r0 += 32) {
    const int i = r0 + lane;
    const int e = i < s1 ? sid[i] : -1;
    const bool ok = i < s1 && (unsigned)e < (unsigned)E;
    const unsigned active = __ballot_sync(kFull, ok);
    if (ok) {
      const unsigned peers = __match_any_sync(active, e);
      const int v = my[e] + __popc(peers & lanemask_lt());
      __syncwarp(active);
      if (lane == __ffs(peers) - 1) my[e] = v + __popc(peers);
      sdst[i] = v;
    }
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kPdThreads) {  // warp counts -> bases
    int acc = pre[e];
    for (int q = 0; q < kPdWarps; ++q) {
      const int v = wh[q * E + e];
      wh[q * E + e] = acc;
      acc += v;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kPdThreads) {  // place
    const int e = sid[i];
    int64_t dst = -1;
    if ((unsigned)e < (unsigned)E) dst = (int64_t)off[e] + wh[(i / chunk) * E + e] + sdst[i];
    if (dst >= P.N) {  // in range by construction; guards a corrupted tile table
      report(P.hdr, MOE_ERR_DEVICE_RANGE, (int)(dst > INT32_MAX ? INT32_MAX : dst));
      dst = -1;
    }
    sdst[i] = (int32_t)dst;
    P.dst_pos[(size_t)a0 * k + i] = (int32_t)dst;
    if (dst >= 0) P.src_idx[dst] = a0 * k + i;
  }
  //    alignment padding rows (a share of them), the previous call's table
  //    (a share), and the table flip by the last CTA
  if (P.align > 1) {
    const int64_t per = (P.N + gridDim.x - 1) / gridDim.x;
    const int64_t r0 = (int64_t)blockIdx.x * per, r1 = min(P.N, r0 + per);
    for (int64_t p = r0 + threadIdx.x; p < r1; p += kPdThreads) {
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
  for (size_t q = (size_t)blockIdx.x * kPdThreads + threadIdx.x; q < oth_used;
       q += (size_t)gridDim.x * kPdThreads)
    oth[q] = 0u;
  __syncthreads();  // sdst holds every row of the range; this CTA is done with the tables
  if (threadIdx.x == 0) {
    if (atomicAdd(&P.hdr->done, 1u) == gridDim.x - 1u) {
      P.hdr->words_used[cur_b] = (uint32_t)((size_t)P.G * E);
      P.hdr->words_used[oth_b] = 0u;
      P.hdr->done = 0u;
      P.hdr->epoch = epoch + 1u;
    }
  }

  // 3. the rows: pipeline w, one bulk load and k bulk stores per token
  if (w >= kPdPipes || lane != 0) return;
  const uint64_t pol = l2_evict_first_policy();
  uint32_t parity = 0;  // bit s: the phase stage s completes next
  int j = 0;
  for (; j < cnt; ++j) {
    const int s = j % stages;
    if (!mbar_wait_bounded(&bars[w][s], (parity >> s) & 1u, kPdTimeoutNs)) {
      report(P.hdr, MOE_ERR_DEVICE_TIMEOUT, a0 + w + kPdPipes * j);
      break;
    }
    parity ^= 1u << s;
    const int li = w + kPdPipes * j;  // the token's index in the range
    const unsigned char* src = ring + (size_t)s * row;
    for (int q = 0; q < k; ++q) {
      const int p = sdst[li * k + q];
      if (p < 0) continue;
      if (P.evict_first)  // output larger than L2: its lines go back to DRAM early
        bulk_store_hint(P.out + (size_t)p * row, src, row, pol);
      else
        bulk_store(P.out + (size_t)p * row, src, row);
    }
    bulk_commit();
    if (issued < cnt) {  // refill the stage token j-1 used
      bulk_wait_read<1>();
      issue_load(issued);
      ++issued;
    }
  }
  // after a timeout: the row loads still in flight land before the CTA exits
  for (; j < issued; ++j) {
    const int s = j % stages;
    (void)mbar_wait_bounded(&bars[w][s], (parity >> s) & 1u, kPdTimeoutNs);
    parity ^= 1u << s;
  }
  bulk_wait_all();
}

struct PdGeom {
  int grid, TB, stages;
  size_t smem;
};

bool pd_geom(int T, int E, int k, int H, int capacity, int num_sms, PdGeom* g) {
  const uint32_t row = (uint32_t)H * 2u;
  if (T <= 0 || capacity > 0 || num_sms < 1 || row < 1024u || row > 32768u) return false;
  int grid = num_sms;
  const int TB = (T + grid - 1) / grid;
  // longer ranges spend the rings' shared memory on their ids and ranks (and
  // their placing grows): Skewed dropless, 1776 assignments a range, ran
  // 5 us slower than the place kernel followed by the dispatch kernel
  if ((int64_t)TB * k > kPdMaxAssign) return false;
  grid = (T + TB - 1) / TB;
  const size_t ints = pd_int_words(E, TB, k) * sizeof(int32_t);
  if (ints >= kPdSmemBudget) return false;
  int stages = (int)((kPdSmemBudget - ints) / ((size_t)kPdPipes * row));
  if (stages > kPdMaxStages) stages = kPdMaxStages;
  if (stages < kPdMinStages) return false;
  g->grid = grid;
  g->TB = TB;
  g->stages = stages;
  g->smem = (size_t)kPdPipes * stages * row + ints;
  return true;
}

}  // namespace

bool place_dispatch_fits(int T, int E, int k, int H, int capacity, int num_sms) {
  PdGeom g;
  return T >= kPdMinTokens && pd_geom(T, E, k, H, capacity, num_sms, &g);
}

cudaError_t launch_place_dispatch(const LaunchEnv& env, const int32_t* ids, const void* x, int T,
                                  int H, int E, int k, int R, int align, int64_t N,
                                  uint32_t* tables, size_t half_words, WsHeader* hdr,
                                  int32_t* counts, int32_t* expert_off, int32_t* rank_off,
                                  int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx,
                                  void* out) {
  PdGeom g;
  if (!pd_geom(T, E, k, H, 0, env.num_sms, &g)) return cudaErrorInvalidValue;
  const TileGeom tiles = layout_tiles(T);
  PdParams P;
  P.ids = ids;
  P.x = static_cast<const char*>(x);
  P.T = T;
  P.E = E;
  P.k = k;
  P.R = R;
  P.align = align;
  P.G = tiles.G;
  P.TT = tiles.TT;
  P.TB = g.TB;
  P.stages = g.stages;
  P.row = (uint32_t)H * 2u;
  P.evict_first = ((int64_t)T * k * H * 2 > (int64_t)192 << 20) ? 1 : 0;
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
  P.out = static_cast<char*>(out);
  int per_sm = 1;  // (raises the kernel's dynamic shared-memory limit to smem)
  const cudaError_t err = blocks_per_sm(reinterpret_cast<const void*>(place_dispatch_kernel),
                                        kPdThreads, g.smem, &per_sm);
  if (err != cudaSuccess) return err;
  return launch_pdl(env, place_dispatch_kernel, dim3((unsigned)g.grid), dim3(kPdThreads), g.smem,
                    P);
}

}  // namespace moe
