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

// Tokens per layout tile (one CTA per tile); the launch doubles it while the
// tiles outnumber the CTAs that fit on the GPU at once.
constexpr int kLayoutTileTokens = 128;

cudaError_t launch_route(const LaunchEnv& env, const float* logits, const float* bias, int T,
                         int E, int k, int renorm, int32_t* ids, float* gates, WsHeader* hdr);

cudaError_t launch_layout(const LaunchEnv& env, const int32_t* ids, int T, int E, int k, int R,
                          int capacity, int align, int64_t N, uint32_t* status, WsHeader* hdr,
                          int32_t* counts, int32_t* expert_off, int32_t* rank_off,
                          int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx,
                          uint64_t timeout_ns);

cudaError_t launch_route_layout(const LaunchEnv& env, const float* logits, const float* bias,
                                int renorm, int32_t* ids, float* gates, int T, int E, int k,
                                int R, int capacity, int align, int64_t N, uint32_t* table,
                                WsHeader* hdr, int32_t* counts, int32_t* expert_off,
                                int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                                int32_t* src_idx, uint64_t timeout_ns);

cudaError_t launch_dispatch_bf16(const LaunchEnv& env, const void* x, const int32_t* dst_pos,
                                 int T, int H, int k, int64_t N, void* out, WsHeader* hdr);

cudaError_t launch_dispatch_fp8(const LaunchEnv& env, const void* x, const int32_t* dst_pos,
                                int T, int H, int k, int64_t N, void* out, float* scales,
                                WsHeader* hdr);

cudaError_t launch_combine(const LaunchEnv& env, const void* y, const int32_t* dst_pos,
                           const float* gates, const void* shared, const void* residual, int T,
                           int H, int k, int64_t N, void* out, WsHeader* hdr);

}  // namespace moe
