// capi.cu -- the C ABI declared in include/moe_route07.h: host-side argument
// checks, workspace sizing, launch and status mapping.  No computation of the
// path happens here; every step runs in the kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "moe_route07.h"

namespace {

using moe::WsHeader;

constexpr size_t kHeaderBytes = sizeof(WsHeader);

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Host-side check of a shape; the limits keep every index in 32 bits.
bool shape_ok(const moe_shape_t* s) {
  if (s == nullptr) return false;
  const int64_t T = s->tokens, H = s->hidden, E = s->experts, k = s->k, R = s->ranks;
  if (T < 0 || H < 8 || (H % 8) != 0) return false;
  if ((s->flags & ~(MOE_F_RENORM | MOE_F_FP8 | MOE_F_SRC_LAYOUT)) != 0u) return false;
  if ((s->flags & MOE_F_FP8) && (H % 128) != 0) return false;
  if (E < 1 || E > 1024 || R < 1 || (E % R) != 0) return false;
  if (k < 1 || k > E || k > 32) return false;
  if (s->capacity < 0 || s->align < 1 || s->align > (1 << 20)) return false;
  if (s->capacity > 0 && s->align != 1) return false;
  if (T * k >= (int64_t(1) << 30)) return false;
  const int64_t segs = (s->flags & MOE_F_SRC_LAYOUT) ? R * E : E;  // R*E <= 2^20
  const int64_t rows = s->capacity > 0 ? segs * s->capacity : T * k + segs * (s->align - 1);
  if (rows >= (int64_t(1) << 31)) return false;
  if (T * (H / 8) >= (int64_t(1) << 31)) return false;
  return true;
}

bool src_layout(const moe_shape_t* s) { return (s->flags & MOE_F_SRC_LAYOUT) != 0u; }

int64_t rows_of(const moe_shape_t* s) {
  const int64_t segs = src_layout(s) ? int64_t(s->ranks) * s->experts : int64_t(s->experts);
  return s->capacity > 0 ? segs * s->capacity
                         : int64_t(s->tokens) * s->k + segs * (s->align - 1);
}

// Workspace: header, then two tile tables of equal size (words a multiple of
// 4); for the per-source-rank layout, header + part counts + kept prefix.
size_t ws_bytes_of(const moe_shape_t* s) {
  if (src_layout(s))
    return kHeaderBytes + (moe::layout_src_part_words(s->tokens, s->experts, s->ranks) +
                           moe::layout_src_cum_words(s->experts, s->ranks)) *
                              sizeof(int32_t);
  const size_t words = (moe::layout_table_words(s->tokens, s->experts) + 3) / 4 * 4;
  return kHeaderBytes + 2 * words * sizeof(uint32_t);
}

size_t half_words_of(size_t ws_bytes) { return ((ws_bytes - kHeaderBytes) / 8) / 4 * 4; }

moe_status_t ws_ok(const moe_shape_t* s, void* ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned(ws, 16)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < ws_bytes_of(s)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    n = 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

moe::LaunchEnv env_of(moe_stream_t stream) {
  moe::LaunchEnv env;
  env.stream = reinterpret_cast<cudaStream_t>(stream);
  env.num_sms = sm_count();
  return env;
}

moe_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned, too small or not zeroed";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE_RANGE: return "device: index out of range";
    case MOE_ERR_DEVICE_TIMEOUT: return "device: bounded wait gave up";
    case MOE_ERR_DEVICE_NAN: return "device: NaN routing key";
  }
  return "unknown status";
}

int64_t moe_layout_rows(const moe_shape_t* shape) {
  if (!shape_ok(shape)) return -1;
  return rows_of(shape);
}

size_t moe_workspace_bytes(const moe_shape_t* shape) {
  if (!shape_ok(shape)) return 0;
  return ws_bytes_of(shape);
}

moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (ws == nullptr || !aligned(ws, 16) || ws_bytes < kHeaderBytes) return MOE_ERR_WORKSPACE;
  return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_route(const moe_shape_t* shape, const float* logits, const float* bias,
                       int32_t* ids, float* gates, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  if (!shape_ok(shape)) return MOE_ERR_INVALID_ARG;
  if (shape->tokens > 0 && (logits == nullptr || ids == nullptr || gates == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(logits, 4) || !aligned(bias, 4) || !aligned(ids, 4) || !aligned(gates, 4))
    return MOE_ERR_INVALID_ARG;
  moe_status_t st = ws_ok(shape, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (shape->tokens == 0) return MOE_OK;
  return from_cuda(moe::launch_route(env_of(stream), logits, bias, shape->tokens,
                                     shape->experts, shape->k,
                                     (shape->flags & MOE_F_RENORM) ? 1 : 0, ids, gates,
                                     static_cast<WsHeader*>(ws)));
}

moe_status_t moe_route_limited(const moe_shape_t* shape, const float* logits, const float* bias,
                               int32_t max_ranks, int32_t* ids, float* gates, void* ws,
                               size_t ws_bytes, moe_stream_t stream) {
  if (!shape_ok(shape) || max_ranks < 1) return MOE_ERR_INVALID_ARG;
  const int R = shape->ranks, Er = shape->experts / shape->ranks;
  if (max_ranks < R && shape->k > (int64_t)max_ranks * Er) return MOE_ERR_INVALID_ARG;
  if (shape->tokens > 0 && (logits == nullptr || ids == nullptr || gates == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(logits, 4) || !aligned(bias, 4) || !aligned(ids, 4) || !aligned(gates, 4))
    return MOE_ERR_INVALID_ARG;
  moe_status_t st = ws_ok(shape, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (shape->tokens == 0) return MOE_OK;
  return from_cuda(moe::launch_route(env_of(stream), logits, bias, shape->tokens,
                                     shape->experts, shape->k,
                                     (shape->flags & MOE_F_RENORM) ? 1 : 0, ids, gates,
                                     static_cast<WsHeader*>(ws), nullptr, 0, R,
                                     max_ranks < R ? max_ranks : 0));
}

moe_status_t moe_layout_remote_first(const moe_shape_t* shape, const int32_t* ids,
                                     int32_t home_rank, int32_t* counts, int32_t* expert_off,
                                     int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                                     int32_t* src_idx, int32_t* tile_expert, void* ws,
                                     size_t ws_bytes, moe_stream_t stream) {
  if (!shape_ok(shape) || src_layout(shape)) return MOE_ERR_INVALID_ARG;
  if (home_rank < 0 || home_rank >= shape->ranks) return MOE_ERR_INVALID_ARG;
  const int64_t N = rows_of(shape);
  if (counts == nullptr || expert_off == nullptr || rank_off == nullptr ||
      rank_counts == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (shape->tokens > 0 && (ids == nullptr || dst_pos == nullptr)) return MOE_ERR_INVALID_ARG;
  if (N > 0 && src_idx == nullptr) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {ids, counts, expert_off, rank_off, rank_counts, dst_pos, src_idx,
                        tile_expert};
  for (const void* p : ptrs)
    if (!aligned(p, 4)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = ws_ok(shape, ws, ws_bytes);
  if (st != MOE_OK) return st;
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  uint32_t* tables = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + kHeaderBytes);
  return from_cuda(moe::launch_layout(env_of(stream), ids, shape->tokens, shape->experts,
                                      shape->k, shape->ranks, shape->capacity, shape->align, N,
                                      tables, half_words_of(ws_bytes), hdr, counts, expert_off,
                                      rank_off, rank_counts, dst_pos, src_idx, true, home_rank,
                                      tile_expert));
}

moe_status_t moe_route_round_robin(const moe_shape_t* shape, int32_t* ids, float* gates,
                                   moe_stream_t stream) {
  if (!shape_ok(shape)) return MOE_ERR_INVALID_ARG;
  if (shape->tokens > 0 && (ids == nullptr || gates == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned(ids, 4) || !aligned(gates, 4)) return MOE_ERR_INVALID_ARG;
  if (shape->tokens == 0) return MOE_OK;
  return from_cuda(moe::launch_route_round_robin(env_of(stream), shape->tokens, shape->experts,
                                                 shape->k, ids, gates));
}

moe_status_t moe_bias_update(const moe_shape_t* shape, const int32_t* counts, float gamma,
                             float* bias, moe_stream_t stream) {
  if (!shape_ok(shape) || counts == nullptr || bias == nullptr) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(gamma) || gamma < 0.0f) return MOE_ERR_INVALID_ARG;
  if (!aligned(counts, 4) || !aligned(bias, 4)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_bias_update(env_of(stream), counts, shape->experts,
                                           int64_t(shape->tokens) * shape->k, gamma, bias));
}

moe_status_t moe_layout(const moe_shape_t* shape, const int32_t* ids, int32_t* counts,
                        int32_t* expert_off, int32_t* rank_off, int32_t* rank_counts,
                        int32_t* dst_pos, int32_t* src_idx, void* ws, size_t ws_bytes,
                        moe_stream_t stream) {
  if (!shape_ok(shape) || src_layout(shape)) return MOE_ERR_INVALID_ARG;
  const int64_t N = rows_of(shape);
  if (counts == nullptr || expert_off == nullptr || rank_off == nullptr ||
      rank_counts == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (shape->tokens > 0 && (ids == nullptr || dst_pos == nullptr)) return MOE_ERR_INVALID_ARG;
  if (N > 0 && src_idx == nullptr) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {ids, counts, expert_off, rank_off, rank_counts, dst_pos, src_idx};
  for (const void* p : ptrs)
    if (!aligned(p, 4)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = ws_ok(shape, ws, ws_bytes);
  if (st != MOE_OK) return st;
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  uint32_t* tables = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + kHeaderBytes);
  return from_cuda(moe::launch_layout(env_of(stream), ids, shape->tokens, shape->experts,
                                      shape->k, shape->ranks, shape->capacity, shape->align, N,
                                      tables, half_words_of(ws_bytes), hdr, counts, expert_off,
                                      rank_off, rank_counts, dst_pos, src_idx, true));
}

moe_status_t moe_layout_src(const moe_shape_t* shape, const int32_t* ids, int32_t* src_counts,
                            int32_t* seg_off, int32_t* pair_counts, int32_t* rank_off,
                            int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx, void* ws,
                            size_t ws_bytes, moe_stream_t stream) {
  if (!shape_ok(shape) || !src_layout(shape)) return MOE_ERR_INVALID_ARG;
  const int64_t N = rows_of(shape);
  if (src_counts == nullptr || seg_off == nullptr || pair_counts == nullptr ||
      rank_off == nullptr || rank_counts == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (shape->tokens > 0 && (ids == nullptr || dst_pos == nullptr)) return MOE_ERR_INVALID_ARG;
  if (N > 0 && src_idx == nullptr) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {ids, src_counts, seg_off, pair_counts, rank_off, rank_counts, dst_pos,
                        src_idx};
  for (const void* p : ptrs)
    if (!aligned(p, 4)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = ws_ok(shape, ws, ws_bytes);
  if (st != MOE_OK) return st;
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  int32_t* partc = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + kHeaderBytes);
  int32_t* scratch =
      partc + moe::layout_src_part_words(shape->tokens, shape->experts, shape->ranks);
  return from_cuda(moe::launch_layout_src(env_of(stream), ids, shape->tokens, shape->experts,
                                          shape->k, shape->ranks, shape->capacity, shape->align,
                                          N, partc, scratch, hdr, src_counts, seg_off,
                                          pair_counts, rank_off, rank_counts, dst_pos,
                                          src_idx));
}

}  // extern "C"

namespace {

// The argument checks of moe_route_layout (and of the route and layout part of
// moe_route_layout_dispatch).
moe_status_t route_layout_args_ok(const moe_shape_t* shape, const float* logits, const float* bias,
                                  int32_t* ids, float* gates, int32_t* counts,
                                  int32_t* expert_off, int32_t* rank_off, int32_t* rank_counts,
                                  int32_t* dst_pos, int32_t* src_idx, void* ws, size_t ws_bytes) {
  if (!shape_ok(shape) || src_layout(shape)) return MOE_ERR_INVALID_ARG;
  const int64_t N = rows_of(shape);
  if (counts == nullptr || expert_off == nullptr || rank_off == nullptr ||
      rank_counts == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (shape->tokens > 0 && (logits == nullptr || ids == nullptr || gates == nullptr ||
                            dst_pos == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (N > 0 && src_idx == nullptr) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {logits, bias, ids, gates, counts, expert_off, rank_off, rank_counts,
                        dst_pos, src_idx};
  for (const void* p : ptrs)
    if (!aligned(p, 4)) return MOE_ERR_INVALID_ARG;
  return ws_ok(shape, ws, ws_bytes);
}

}  // namespace

extern "C" {

moe_status_t moe_route_layout(const moe_shape_t* shape, const float* logits, const float* bias,
                              int32_t* ids, float* gates, int32_t* counts, int32_t* expert_off,
                              int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                              int32_t* src_idx, void* ws, size_t ws_bytes, moe_stream_t stream) {
  const moe_status_t st = route_layout_args_ok(shape, logits, bias, ids, gates, counts,
                                               expert_off, rank_off, rank_counts, dst_pos,
                                               src_idx, ws, ws_bytes);
  if (st != MOE_OK) return st;
  const int64_t N = rows_of(shape);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  uint32_t* tables = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + kHeaderBytes);
  const size_t half = half_words_of(ws_bytes);
  const moe::LaunchEnv env = env_of(stream);
  if (moe::route_layout_small_fits(shape->tokens, shape->experts, shape->k))
    return from_cuda(moe::launch_route_layout_small(
        env, logits, bias, shape->tokens, shape->experts, shape->k, shape->ranks,
        (shape->flags & MOE_F_RENORM) ? 1 : 0, shape->capacity, shape->align, N, hdr, ids, gates,
        counts, expert_off, rank_off, rank_counts, dst_pos, src_idx));
  if (shape->tokens > 0) {
    const cudaError_t err = moe::launch_route(env, logits, bias, shape->tokens, shape->experts,
                                              shape->k, (shape->flags & MOE_F_RENORM) ? 1 : 0,
                                              ids, gates, hdr, tables, half);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  }
  return from_cuda(moe::launch_layout(env, ids, shape->tokens, shape->experts, shape->k,
                                      shape->ranks, shape->capacity, shape->align, N, tables, half,
                                      hdr, counts, expert_off, rank_off, rank_counts, dst_pos,
                                      src_idx, false));
}

moe_status_t moe_route_layout_dispatch(const moe_shape_t* shape, const float* logits,
                                       const float* bias, const void* x, int32_t* ids,
                                       float* gates, int32_t* counts, int32_t* expert_off,
                                       int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                                       int32_t* src_idx, void* out, float* scales, void* ws,
                                       size_t ws_bytes, moe_stream_t stream) {
  if (!shape_ok(shape) || src_layout(shape)) return MOE_ERR_INVALID_ARG;
  const bool fp8 = (shape->flags & MOE_F_FP8) != 0u;
  if (shape->tokens > 0 && (x == nullptr || out == nullptr || (fp8 && scales == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(scales, 4)) return MOE_ERR_INVALID_ARG;
  const int T = shape->tokens, E = shape->experts, k = shape->k, H = shape->hidden;
  if (!fp8 && T > 0 && !moe::route_layout_small_fits(T, E, k)) {
    const moe::LaunchEnv env = env_of(stream);
    if (moe::place_dispatch_fits(T, E, k, H, shape->capacity, env.num_sms)) {
      // the route kernel fills the tile table; one kernel places and streams the rows
      const moe_status_t sa = route_layout_args_ok(shape, logits, bias, ids, gates, counts,
                                                   expert_off, rank_off, rank_counts, dst_pos,
                                                   src_idx, ws, ws_bytes);
      if (sa != MOE_OK) return sa;
      WsHeader* hdr = static_cast<WsHeader*>(ws);
      uint32_t* tables = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + kHeaderBytes);
      const size_t half = half_words_of(ws_bytes);
      const cudaError_t err =
          moe::launch_route(env, logits, bias, T, E, k, (shape->flags & MOE_F_RENORM) ? 1 : 0,
                            ids, gates, hdr, tables, half);
      if (err != cudaSuccess) return MOE_ERR_CUDA;
      return from_cuda(moe::launch_place_dispatch(
          env, ids, x, T, H, E, k, shape->ranks, shape->align, rows_of(shape), tables, half, hdr,
          counts, expert_off, rank_off, rank_counts, dst_pos, src_idx, out));
    }
  }
  moe_status_t st = moe_route_layout(shape, logits, bias, ids, gates, counts, expert_off,
                                     rank_off, rank_counts, dst_pos, src_idx, ws, ws_bytes,
                                     stream);
  if (st != MOE_OK || shape->tokens == 0) return st;
  const moe::LaunchEnv env = env_of(stream);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  const int64_t N = rows_of(shape);
  if (fp8)
    return from_cuda(moe::launch_dispatch_fp8(env, x, dst_pos, shape->tokens, shape->hidden,
                                              shape->k, N, out, scales, hdr));
  return from_cuda(moe::launch_dispatch_bf16(env, x, dst_pos, shape->tokens, shape->hidden,
                                             shape->k, N, out, hdr, true));
}

moe_status_t moe_dispatch(const moe_shape_t* shape, const void* x, const int32_t* dst_pos,
                          void* out, float* scales, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  if (!shape_ok(shape)) return MOE_ERR_INVALID_ARG;
  const bool fp8 = (shape->flags & MOE_F_FP8) != 0u;
  if (shape->tokens > 0 && (x == nullptr || dst_pos == nullptr || out == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (fp8 && shape->tokens > 0 && scales == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(dst_pos, 4) || !aligned(scales, 4))
    return MOE_ERR_INVALID_ARG;
  moe_status_t st = ws_ok(shape, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (shape->tokens == 0) return MOE_OK;
  const moe::LaunchEnv env = env_of(stream);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  const int64_t N = rows_of(shape);
  if (fp8)
    return from_cuda(moe::launch_dispatch_fp8(env, x, dst_pos, shape->tokens, shape->hidden,
                                              shape->k, N, out, scales, hdr));
  return from_cuda(moe::launch_dispatch_bf16(env, x, dst_pos, shape->tokens, shape->hidden,
                                             shape->k, N, out, hdr));
}

moe_status_t moe_combine(const moe_shape_t* shape, const void* y, const int32_t* dst_pos,
                         const float* gates, const void* shared, const void* residual,
                         void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!shape_ok(shape)) return MOE_ERR_INVALID_ARG;
  if (shape->tokens > 0 &&
      (y == nullptr || dst_pos == nullptr || gates == nullptr || out == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(out, 16) || !aligned(shared, 16) || !aligned(residual, 16) ||
      !aligned(dst_pos, 4) || !aligned(gates, 4))
    return MOE_ERR_INVALID_ARG;
  moe_status_t st = ws_ok(shape, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (shape->tokens == 0) return MOE_OK;
  return from_cuda(moe::launch_combine(env_of(stream), y, dst_pos, gates, shared, residual,
                                       shape->tokens, shape->hidden, shape->k, rows_of(shape),
                                       out, static_cast<WsHeader*>(ws), shape->capacity > 0));
}

moe_status_t moe_selftest_wait_timeout(void* ws, uint32_t timeout_us, moe_stream_t stream) {
  if (ws == nullptr || !aligned(ws, 16)) return MOE_ERR_WORKSPACE;
  if (timeout_us < 1u || timeout_us > 2000000u) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_wait_timeout_selftest(env_of(stream), static_cast<WsHeader*>(ws),
                                                     uint64_t(timeout_us) * 1000u));
}

moe_status_t moe_get_device_error(void* ws, int32_t* detail, moe_stream_t stream) {
  if (ws == nullptr || !aligned(ws, 16)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t h[2] = {0, 0};
  if (cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (h[0] != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof(h), s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (detail != nullptr) *detail = h[1];
  return static_cast<moe_status_t>(h[0]);
}

}  // extern "C"
