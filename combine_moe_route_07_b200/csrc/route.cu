// route.cu -- step 1: one warp per token (see route_core.cuh).  With a tile
// table the kernel also counts the routed ids per layout tile: each CTA's
// shared-memory histogram of its 8 tokens is added into the table row of the
// tile those tokens belong to (integer adds, so the counts do not depend on
// the order the CTAs run in).  That table is the first half of moe_layout.
#include "common.cuh"
#include "kernels.h"
#include "route_core.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;  // tokens per CTA step

template <int NK, bool HIST>
__global__ void __launch_bounds__(kThreads)
    route_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E,
                 int k, int renorm, int32_t* __restrict__ ids, float* __restrict__ gates,
                 WsHeader* hdr, uint32_t* __restrict__ tables, int TT, size_t table_words) {
  extern __shared__ int32_t hist[];  // [E] (HIST)
  __shared__ uint32_t cand_all[kWarps][NK >= 8 ? 3 * kMaxCand : 1];
  pdl_wait();  // logits (and the tile table) may come from the kernel launched before
  pdl_trigger();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float b[NK];
  load_bias<NK>(bias, E, lane, b);
  uint32_t* tab = nullptr;
  if constexpr (HIST) {
    const uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(&hdr->epoch);
    tab = tables + (size_t)(epoch & 1u) * table_words;
    for (int e = threadIdx.x; e < E; e += kThreads) hist[e] = 0;
    __syncthreads();
  }
  for (int g0 = blockIdx.x * kWarps; g0 < T; g0 += gridDim.x * kWarps) {
    const int t = g0 + w;
    if (t < T) {
      int tok[1] = {t}, e[1];
      float g[1];
      int nan_tok;
      if constexpr (NK >= 8)
        nan_tok = route_token_thr<NK>(logits, t, T, b, E, k, renorm, lane, cand_all[w], e[0], g[0]);
      else
        nan_tok = route_tokens<NK, 1>(logits, tok, T, b, E, k, renorm, lane, e, g);
      if (nan_tok >= 0 && lane == 0) report(hdr, MOE_ERR_DEVICE_NAN, nan_tok);
      if (lane < k) {
        ids[(size_t)t * k + lane] = e[0];
        gates[(size_t)t * k + lane] = g[0];
        if constexpr (HIST) atomicAdd(&hist[e[0]], 1);
      }
    }
    if constexpr (HIST) {  // the 8 tokens lie in one tile (TT is a multiple of 8)
      __syncthreads();
      uint32_t* row = tab + (size_t)(g0 / TT) * E;
      for (int e = threadIdx.x; e < E; e += kThreads) {
        const int c = hist[e];
        if (c != 0) {
          atomicAdd(row + e, (uint32_t)c);
          hist[e] = 0;
        }
      }
      __syncthreads();
    }
  }
}

template <int NK, bool HIST>
cudaError_t launch_nk(const LaunchEnv& env, const float* logits, const float* bias, int T, int E,
                      int k, int renorm, int32_t* ids, float* gates, WsHeader* hdr,
                      uint32_t* tables, int TT, size_t table_words) {
  auto kern = route_kernel<NK, HIST>;
  const size_t smem = HIST ? (size_t)E * sizeof(int32_t) : 0;
  int per_sm = 1;
  const cudaError_t err = blocks_per_sm(reinterpret_cast<const void*>(kern), kThreads, smem, &per_sm);
  if (err != cudaSuccess) return err;
  int64_t blocks = ((int64_t)T + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)per_sm * env.num_sms;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_pdl(env, kern, dim3((unsigned)blocks), dim3(kThreads), smem, logits, bias, T, E,
                    k, renorm, ids, gates, hdr, tables, TT, table_words);
}

template <bool HIST>
cudaError_t launch_any(const LaunchEnv& env, const float* logits, const float* bias, int T, int E,
                       int k, int renorm, int32_t* ids, float* gates, WsHeader* hdr,
                       uint32_t* tables, int TT, size_t table_words) {
  const int nk = (E + 31) / 32;
#define MOE_ROUTE_NK(N)                                                                         \
  if (nk <= N)                                                                                  \
    return launch_nk<N, HIST>(env, logits, bias, T, E, k, renorm, ids, gates, hdr, tables, TT, \
                              table_words);
  MOE_ROUTE_NK(1)
  MOE_ROUTE_NK(2)
  MOE_ROUTE_NK(4)
  MOE_ROUTE_NK(8)
  MOE_ROUTE_NK(16)
#undef MOE_ROUTE_NK
  return launch_nk<32, HIST>(env, logits, bias, T, E, k, renorm, ids, gates, hdr, tables, TT,
                             table_words);
}

}  // namespace

cudaError_t launch_route(const LaunchEnv& env, const float* logits, const float* bias, int T,
                         int E, int k, int renorm, int32_t* ids, float* gates, WsHeader* hdr,
                         uint32_t* tables, size_t half_words) {
  if (tables == nullptr)
    return launch_any<false>(env, logits, bias, T, E, k, renorm, ids, gates, hdr, nullptr, 1, 0);
  const TileGeom geom = layout_tiles(T);
  return launch_any<true>(env, logits, bias, T, E, k, renorm, ids, gates, hdr, tables, geom.TT,
                          half_words);
}

}  // namespace moe
