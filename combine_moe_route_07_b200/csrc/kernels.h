// kernels.h -- internal launch interface between the C ABI (capi.cu) and the
// kernels.  Not installed; the public interface is include/moe_route07.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

struct WsHeader;

struct LaunchEnv {
  cudaStream_t stream;
  int num_sms;
};

// Launch `kernel` on env.stream with programmatic stream serialization, so
// its CTAs may start while the previous kernel drains (the kernel calls
// pdl_wait() before touching anything the previous kernel wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(const LaunchEnv& env, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                       size_t smem, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = env.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Resident CTAs per SM (at least 1) of `kernel` at this block size and
// dynamic shared memory on the current device, after raising the kernel's
// dynamic shared-memory limit to at least `smem` (when smem > 0).  Every
// launch of a kernel with dynamic shared memory above 48 KiB less its static
// shared memory must come through here first.  Both
// are cached per (device, kernel, threads, smem): the runtime's occupancy
// query costs host time that would otherwise be paid on every launch.
cudaError_t blocks_per_sm(const void* kernel, int threads, size_t smem, int* out);

// Layout tiles: runs of TT consecutive tokens, TT a multiple of
// kLayoutTileQuantum, at most kLayoutMaxTiles of them.  The workspace holds
// two tables (used on alternate calls) of one row of E counters per tile.
constexpr int kLayoutTileQuantum = 16;
constexpr int kLayoutMaxTiles = 128;

struct TileGeom {
  int TT;  // tokens per tile
  int G;   // tiles
};
inline TileGeom layout_tiles(int T) {
  TileGeom g;
  const int64_t q = kLayoutTileQuantum;
  int64_t want = T > 0 ? (T + q - 1) / q : 1;
  if (want > kLayoutMaxTiles) want = kLayoutMaxTiles;
  int64_t tt = T > 0 ? (T + want - 1) / want : q;
  tt = ((tt + q - 1) / q) * q;
  g.TT = (int)tt;
  g.G = T > 0 ? (int)((T + tt - 1) / tt) : 1;
  return g;
}
// Words in one of the two tile tables for T tokens and E experts.
inline size_t layout_table_words(int T, int E) {
  int64_t rows = T > 0 ? ((int64_t)T + kLayoutTileQuantum - 1) / kLayoutTileQuantum : 1;
  if (rows > kLayoutMaxTiles) rows = kLayoutMaxTiles;
  return (size_t)rows * (size_t)E;
}

// Per-source-rank layout geometry: R source shards of Ts consecutive tokens,
// each cut into P parts of TP tokens (about 256 parts in all, at least 16
// tokens each); one CTA per part counts and later places its assignments.
struct SrcGeom {
  int Ts;  // tokens per shard
  int TP;  // tokens per part
  int P;   // parts per shard
};
inline SrcGeom layout_src_geom(int T, int R) {
  SrcGeom g;
  g.Ts = T > 0 ? (T + R - 1) / R : 1;
  int want = 256 / R;
  if (want < 1) want = 1;
  int tp = (g.Ts + want - 1) / want;
  if (tp < 16) tp = 16;
  g.TP = tp;
  g.P = (g.Ts + tp - 1) / tp;
  return g;
}
// Workspace words after the header: part counts [R][P][E], then the
// per-segment totals [R*E], the exclusive prefix of kept rows over the R*E
// segments (+1) and one 64-bit sum per chunk of 1024 segments.
inline size_t layout_src_part_words(int T, int E, int R) {
  const SrcGeom g = layout_src_geom(T, R);
  return ((size_t)R * g.P * E + 3) / 4 * 4;
}
inline size_t layout_src_cum_words(int E, int R) {
  const size_t chunks = ((size_t)R * E + 1023) / 1024;
  return ((size_t)R * E + 3) / 4 * 4 + ((size_t)R * E + 1 + 3) / 4 * 4 + (2 * chunks + 3) / 4 * 4;
}

// Per-source-rank layout: count parts, reduce, scan segments, place (four
// kernels chained by PDL).  partc (layout_src_part_words) and scratch
// (layout_src_cum_words) are workspace.
cudaError_t launch_layout_src(const LaunchEnv& env, const int32_t* ids, int T, int E, int k, int R,
                              int capacity, int align, int64_t N, int32_t* partc,
                              int32_t* scratch, WsHeader* hdr, int32_t* src_counts,
                              int32_t* seg_off, int32_t* pair_counts, int32_t* rank_off,
                              int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx);

// tables != nullptr: also add each routed token's ids into the layout tile
// table the next place pass reads (the fused route + layout path).  `tables`
// holds two tables of `half_words` words each.  0 < max_ranks < R: each
// token's experts come from at most max_ranks of the R ranks.
cudaError_t launch_route(const LaunchEnv& env, const float* logits, const float* bias, int T,
                         int E, int k, int renorm, int32_t* ids, float* gates, WsHeader* hdr,
                         uint32_t* tables = nullptr, size_t half_words = 0, int R = 1,
                         int max_ranks = 0);

// Layout of `ids` (count pass + place pass).  count_ids == false: the tile
// table was already filled by a route launch with tables (fused path).
// 0 <= home < R: rank slices in the order home+1, ..., home (remote first);
// otherwise the natural order.  tile_expert (or nullptr): the expert of each
// align-row tile, -1 past the rows used.
cudaError_t launch_layout(const LaunchEnv& env, const int32_t* ids, int T, int E, int k, int R,
                          int capacity, int align, int64_t N, uint32_t* tables,
                          size_t half_words, WsHeader* hdr, int32_t* counts, int32_t* expert_off,
                          int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                          int32_t* src_idx, bool count_ids = true, int home = -1,
                          int32_t* tile_expert = nullptr);

// x_ready: x is not written by the kernel launched just before and every
// earlier kernel has finished (the case right behind this library's layout
// kernels), so x rows may be fetched before waiting on that kernel.
cudaError_t launch_dispatch_bf16(const LaunchEnv& env, const void* x, const int32_t* dst_pos,
                                 int T, int H, int k, int64_t N, void* out, WsHeader* hdr,
                                 bool x_ready = false);

cudaError_t launch_dispatch_fp8(const LaunchEnv& env, const void* x, const int32_t* dst_pos,
                                int T, int H, int k, int64_t N, void* out, float* scales,
                                WsHeader* hdr);

// Self-test of the bounded-wait error path: a wait that nothing completes.
cudaError_t launch_wait_timeout_selftest(const LaunchEnv& env, WsHeader* hdr,
                                         uint64_t timeout_ns);

// Steps 1-3 for a small batch in one launch of one thread-block cluster
// (decode-sized): at most kSmallMaxAssign assignments and kSmallMaxExperts
// experts.  Same results as launch_route + launch_layout.  The cluster routes
// on 8 SMs, one warp per token: at 128 tokens x 8 it saves a launch over the
// two kernels; by 256 x 8 the two kernels' wider route has caught up.
constexpr int kSmallMaxAssign = 1024;
constexpr int kSmallMaxExperts = 512;
bool route_layout_small_fits(int T, int E, int k);
cudaError_t launch_route_layout_small(const LaunchEnv& env, const float* logits,
                                      const float* bias, int T, int E, int k, int R, int renorm,
                                      int capacity, int align, int64_t N, WsHeader* hdr,
                                      int32_t* ids, float* gates, int32_t* counts,
                                      int32_t* expert_off, int32_t* rank_off,
                                      int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx);

// Steps 3-4 behind a route launch with the tile table (the fused steps 1-4,
// bf16, dropless, at least kPdMinTokens tokens, rows of 1-32 KiB, at most 512
// assignments a CTA): each CTA
// places a contiguous range of tokens from the tile table and streams their
// rows by bulk copy.  Same results as launch_layout (count_ids = false) +
// launch_dispatch_bf16.  place_dispatch_fits says whether a batch fits.
constexpr int kPdMinTokens = 2048;
bool place_dispatch_fits(int T, int E, int k, int H, int capacity, int num_sms);
cudaError_t launch_place_dispatch(const LaunchEnv& env, const int32_t* ids, const void* x, int T,
                                  int H, int E, int k, int R, int align, int64_t N,
                                  uint32_t* tables, size_t half_words, WsHeader* hdr,
                                  int32_t* counts, int32_t* expert_off, int32_t* rank_off,
                                  int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx,
                                  void* out);

// Round-robin router (diagnostic): ids[t,j] = (t*k + j) mod E, gates 1/k.
cudaError_t launch_route_round_robin(const LaunchEnv& env, int T, int E, int k, int32_t* ids,
                                     float* gates);

// b_e += gamma * sign(assignments/E - counts[e]) for the E experts, in place.
cudaError_t launch_bias_update(const LaunchEnv& env, const int32_t* counts, int E,
                               int64_t assignments, float gamma, float* bias);

// sparse: most slots may be dropped (capacity mode)
cudaError_t launch_combine(const LaunchEnv& env, const void* y, const int32_t* dst_pos,
                           const float* gates, const void* shared, const void* residual, int T,
                           int H, int k, int64_t N, void* out, WsHeader* hdr, bool sparse);

}  // namespace moe
