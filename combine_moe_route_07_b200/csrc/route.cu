// route.cu -- step 1: one warp per token (see route_core.cuh).  With a tile
// table the kernel also counts the routed ids per layout tile: each CTA
// keeps a shared-memory histogram of the tokens it routed in the current tile
// and adds it into that tile's table row when its tokens move on to the next
// tile (integer adds, so the counts do not depend on the order the CTAs run
// in).  That table is the first half of moe_layout.
//
// Each CTA routes a contiguous run of tokens (a multiple of 8 long), warp w
// the tokens c0 + w, c0 + w + 8, ...; a group of 8 never straddles a tile
// (tiles are multiples of 16 tokens), so the CTA's histogram is flushed at
// most once per tile it touches rather than once per group.
//
// STAGE (many experts per token, rows of 16-byte multiples): each warp keeps
// two or three shared-memory row buffers and prefetches the logits of its
// next one or two tokens by bulk copy (TMA) while it routes the current one,
// so the rows' DRAM latency overlaps the selection arithmetic.  Without a
// rank limit the staged rows go through select_fast (float keys, exact
// fallback to the code form), and with renormalised gates and k <= 16 the
// softmax of two consecutive tokens of a warp runs as one pass.
#include "bulk.cuh"
#include "common.cuh"
#include "kernels.h"
#include "route_core.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;  // tokens per CTA group
constexpr uint64_t kRowTimeoutNs = 1000000000ull;
// STAGE: row buffers per warp.  Three (two rows in flight ahead) for rows of
// up to 256 experts; two for longer rows, whose third buffer would cost a CTA
// per SM (Fine-grained, 512 experts: 75 us with two against 88 with three).
constexpr int row_stages(int nk) { return nk <= 8 ? 3 : 2; }
constexpr int kMaxRowStages = 3;

template <int NK, bool HIST, bool STAGE, bool LIMIT>
__global__ void __launch_bounds__(kThreads, (STAGE && !LIMIT && NK <= 16) ? 4 : 1)
    route_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E,
                 int k, int renorm, int32_t* __restrict__ ids, float* __restrict__ gates,
                 WsHeader* hdr, uint32_t* __restrict__ tables, int TT, size_t table_words,
                 int per, int R, int M) {
  // dynamic: [hist: E int32, padded to 16 B] (HIST), [rows: kWarps x kRowStages x E floats]
  // (STAGE),
  // [rank limit: kWarps x (R + ceil(R/32)) words] (M < R), [bias: E floats] (STAGE)
  extern __shared__ __align__(16) unsigned char dyn[];
  __shared__ __align__(16) uint32_t cand_all[kWarps][NK >= 8 ? 3 * kMaxCand : 1];
  constexpr int kRowStages = row_stages(NK);
  __shared__ uint64_t bars[kWarps][kMaxRowStages];
  int32_t* hist = reinterpret_cast<int32_t*>(dyn);
  const size_t hist_bytes = HIST ? (((size_t)E * 4 + 15) & ~(size_t)15) : 0;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float* buf = reinterpret_cast<float*>(dyn + hist_bytes) + (size_t)w * kRowStages * E;
  RankLimit lim;  // compiled in only for LIMIT (then M < R)
  lim.R = R;
  lim.M = LIMIT ? M : 0;
  lim.init(E, lane);
  const size_t lim_words = lim.on() ? (size_t)R + (R + 31) / 32 : 0;
  uint32_t* lim_base = reinterpret_cast<uint32_t*>(
      dyn + hist_bytes + (STAGE ? (size_t)kWarps * kRowStages * E * sizeof(float) : 0));
  if (lim.on()) lim.smem = lim_base + (size_t)w * lim_words;
  float* sbias = reinterpret_cast<float*>(lim_base + (size_t)kWarps * lim_words);
  if (STAGE && lane == 0) {
    for (int q = 0; q < kRowStages; ++q) mbar_init(&bars[w][q], 1);
    mbar_fence_init();
  }
  __syncwarp();
  pdl_wait();  // logits (and the tile table) may come from the kernel launched before
  pdl_trigger();
  float b[NK];
  if constexpr (!STAGE) load_bias<NK>(bias, E, lane, b);
  FastLanes<STAGE ? NK : 8> fast;  // the staged form without a rank limit
  if constexpr (STAGE && !LIMIT) fast.init(E, lane);
  if constexpr (STAGE) {  // the bias, read per token from shared memory
    for (int e = threadIdx.x; e < E; e += kThreads) sbias[e] = bias != nullptr ? __ldg(bias + e) : 0.0f;
    __syncthreads();
  }
  const int c0 = (int)min((int64_t)blockIdx.x * per, (int64_t)T);
  const int c1 = min(T, c0 + per);
  const int n = (c1 - c0 + kWarps - 1) / kWarps;  // groups: the same for every warp
  uint32_t* tab = nullptr;
  int cur_tile = 0, tile_end = 0;  // the current tile and its first token past the end
  if constexpr (HIST) {
    const uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(&hdr->epoch);
    tab = tables + (size_t)(epoch & 1u) * table_words;
    for (int e = threadIdx.x; e < E; e += kThreads) hist[e] = 0;
    __syncthreads();
    cur_tile = c0 / TT;
    tile_end = (cur_tile + 1) * TT;
  }
  auto flush = [&](int tile) {  // caller: __syncthreads() before and after
    uint32_t* row = tab + (size_t)tile * E;
    for (int e = threadIdx.x; e < E; e += kThreads) {
      const int c = hist[e];
      if (c != 0) {
        atomicAdd(row + e, (uint32_t)c);
        hist[e] = 0;
      }
    }
  };
  // STAGE: buffer i mod kRowStages of this warp holds token c0 + w + 8*i
  uint32_t parity = 0, pending = 0;
  int sb = 0;  // the buffer of the current token
  bool alive = true;
  auto issue = [&](int tok, int q) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[w][q], (uint32_t)E * 4u);
      bulk_load(buf + (size_t)q * E, logits + (size_t)tok * E, (uint32_t)E * 4u, &bars[w][q]);
    }
    pending |= 1u << q;
  };
  if constexpr (STAGE) {
    for (int q = 0; q + 1 < kRowStages; ++q)
      if (c0 + w + kWarps * q < c1) issue(c0 + w + kWarps * q, q);
  }
  // the float-key form with renormalised gates and k <= 16: a token's softmax
  // waits for the warp's next token of that form and the two are done in one
  // pass (the same bits as one at a time); p_t is the waiting token
  const bool pair = STAGE && !LIMIT && renorm && k <= 16;
  int p_t = -1;
  float p_raw = 0.0f;

  for (int i = 0; i < n; ++i) {
    const int g0 = c0 + kWarps * i;
    if constexpr (HIST) {
      if (g0 >= tile_end) {  // (the same for every warp of the CTA)
        __syncthreads();
        flush(cur_tile);
        __syncthreads();
        cur_tile = g0 / TT;
        tile_end = (cur_tile + 1) * TT;
      }
    }
    const int t = g0 + w;
    if (t < c1 && alive) {
      int e1 = 0;
      float g1 = 0.0f;
      int nan_tok;
      bool gate_ready = true;  // false: the softmax waits for the next token
      if constexpr (STAGE) {
        // the buffer before this one was last read for token i-1 (done:
        // __syncwarp below); it takes token i + kRowStages - 1
        const int ahead = t + kWarps * (kRowStages - 1);
        if (ahead < c1) issue(ahead, sb == 0 ? kRowStages - 1 : sb - 1);
        const bool ok = __all_sync(
            kFull, mbar_wait_bounded(&bars[w][sb], (parity >> sb) & 1u, kRowTimeoutNs));
        if (ok) {
          parity ^= 1u << sb;
          pending &= ~(1u << sb);
          const float* srow = buf + (size_t)sb * E;
          if constexpr (LIMIT) {
            nan_tok = route_token_smem<NK, true>(srow, sbias, t, E, k, renorm, lane, cand_all[w],
                                                 e1, g1, lim);
          } else {
            float raw1 = 0.0f;
            nan_tok = -1;
            if (!select_fast<NK>(srow, sbias, bias != nullptr, k, lane, cand_all[w], fast, e1,
                                 raw1)) {
              nan_tok = route_token_exact<NK>(srow, sbias, t, E, k, renorm, lane, cand_all[w],
                                              e1, g1);
            } else if (!pair) {
              g1 = gate_staged(srow, raw1, E, k, renorm, lane);
            } else if (p_t < 0) {
              p_t = t;
              p_raw = raw1;
              gate_ready = false;
            } else {
              float ga;
              gate_renorm_pair(p_raw, raw1, k, lane, ga, g1);
              if (lane < k) gates[(size_t)p_t * k + lane] = ga;
              p_t = -1;
            }
          }
        } else {
          if (lane == 0) report(hdr, MOE_ERR_DEVICE_TIMEOUT, t);
          alive = false;  // routes nothing more; still takes part in the CTA barriers
        }
      } else if constexpr (NK >= 8) {
        nan_tok = route_token_thr<NK>(logits, t, T, b, E, k, renorm, lane, cand_all[w], e1, g1,
                                      lim);
      } else {
        int tok[1] = {t}, ea[1];
        float ga[1];
        nan_tok = route_tokens<NK, 1>(logits, tok, T, b, E, k, renorm, lane, ea, ga, lim);
        e1 = ea[0];
        g1 = ga[0];
      }
      if (alive) {
        if (nan_tok >= 0 && lane == 0) report(hdr, MOE_ERR_DEVICE_NAN, nan_tok);
        if (lane < k) {
          ids[(size_t)t * k + lane] = e1;
          if (gate_ready) gates[(size_t)t * k + lane] = g1;
          if constexpr (HIST) atomicAdd(&hist[e1], 1);
        }
      }
    }
    if constexpr (STAGE) {
      __syncwarp();  // every lane is done with this buffer
      sb = sb + 1 == kRowStages ? 0 : sb + 1;
    }
  }
  if (p_t >= 0) {  // a token whose softmax still waits: alone
    const float g = gate_renorm(p_raw, k, lane);
    if (lane < k) gates[(size_t)p_t * k + lane] = g;
  }
  if constexpr (STAGE) {  // copies still in flight land before the CTA exits
    for (int q = 0; q < kRowStages; ++q)
      if ((pending >> q) & 1u)
        (void)mbar_wait_bounded(&bars[w][q], (parity >> q) & 1u, kRowTimeoutNs);
  }
  if constexpr (HIST) {
    __syncthreads();
    if (n > 0) flush(cur_tile);
  }
}

template <int NK, bool HIST>
cudaError_t launch_nk(const LaunchEnv& env, const float* logits, const float* bias, int T, int E,
                      int k, int renorm, int32_t* ids, float* gates, WsHeader* hdr,
                      uint32_t* tables, int TT, size_t table_words, int R, int M) {
  const size_t hist_bytes = HIST ? (((size_t)E * 4 + 15) & ~(size_t)15) : 0;
  // rows staged by bulk copy: many keys per lane, 16-byte rows and base
  const bool stage = NK >= 8 && (E % 4) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15u) == 0;
  const bool limit = M > 0 && M < R;
  auto kern = stage ? (limit ? route_kernel<NK, HIST, NK >= 8, true>
                             : route_kernel<NK, HIST, NK >= 8, false>)
                    : (limit ? route_kernel<NK, HIST, false, true>
                             : route_kernel<NK, HIST, false, false>);
  const size_t smem = hist_bytes +
                      (stage ? (size_t)kWarps * row_stages(NK) * E * sizeof(float) : 0) +
                      (limit ? (size_t)kWarps * (R + (R + 31) / 32) * sizeof(uint32_t) : 0) +
                      (stage ? (size_t)E * sizeof(float) : 0);
  int per_sm = 1;
  const cudaError_t err = blocks_per_sm(reinterpret_cast<const void*>(kern), kThreads, smem, &per_sm);
  if (err != cudaSuccess) return err;
  int64_t blocks = ((int64_t)T + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)per_sm * env.num_sms;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  // contiguous runs of tokens, a multiple of kWarps long
  int64_t per = ((int64_t)T + blocks - 1) / blocks;
  per = (per + kWarps - 1) / kWarps * kWarps;
  if (per < kWarps) per = kWarps;
  blocks = ((int64_t)T + per - 1) / per;
  if (blocks < 1) blocks = 1;
  return launch_pdl(env, kern, dim3((unsigned)blocks), dim3(kThreads), smem, logits, bias, T, E,
                    k, renorm, ids, gates, hdr, tables, TT, table_words, (int)per, R, M);
}

template <bool HIST>
cudaError_t launch_any(const LaunchEnv& env, const float* logits, const float* bias, int T, int E,
                       int k, int renorm, int32_t* ids, float* gates, WsHeader* hdr,
                       uint32_t* tables, int TT, size_t table_words, int R, int M) {
  const int nk = (E + 31) / 32;
#define MOE_ROUTE_NK(N)                                                                         \
  if (nk <= N)                                                                                  \
    return launch_nk<N, HIST>(env, logits, bias, T, E, k, renorm, ids, gates, hdr, tables, TT, \
                              table_words, R, M);
  MOE_ROUTE_NK(1)
  MOE_ROUTE_NK(2)
  MOE_ROUTE_NK(4)
  MOE_ROUTE_NK(8)
  MOE_ROUTE_NK(16)
#undef MOE_ROUTE_NK
  return launch_nk<32, HIST>(env, logits, bias, T, E, k, renorm, ids, gates, hdr, tables, TT,
                             table_words, R, M);
}

// The round-robin router: ids[t,j] = (t*k + j) mod E, gates 1/k.  "GPU MoE
// all-to-all", section "How to tell whether the all-to-all is your
// bottleneck": swapping the learned router for a uniform round-robin
// assignment separates routing skew from the cost of the exchange itself.
__global__ void __launch_bounds__(kThreads)
    round_robin_kernel(int T, int E, int k, int32_t* __restrict__ ids,
                       float* __restrict__ gates) {
  pdl_wait();  // ids and gates may still be read by the kernel launched before
  pdl_trigger();
  const int64_t n = (int64_t)T * k;
  const float g = (float)(1.0 / (double)k);
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * kThreads) {
    ids[i] = (int32_t)(i % E);  // i = t*k + j
    gates[i] = g;
  }
}

}  // namespace

cudaError_t launch_route_round_robin(const LaunchEnv& env, int T, int E, int k, int32_t* ids,
                                     float* gates) {
  const int64_t n = (int64_t)T * k;
  int64_t grid = (n + kThreads - 1) / kThreads;
  if (grid > 4 * (int64_t)env.num_sms) grid = 4 * (int64_t)env.num_sms;
  if (grid < 1) grid = 1;
  return launch_pdl(env, round_robin_kernel, dim3((unsigned)grid), dim3(kThreads), 0, T, E, k,
                    ids, gates);
}

cudaError_t launch_route(const LaunchEnv& env, const float* logits, const float* bias, int T,
                         int E, int k, int renorm, int32_t* ids, float* gates, WsHeader* hdr,
                         uint32_t* tables, size_t half_words, int R, int max_ranks) {
  if (tables == nullptr)
    return launch_any<false>(env, logits, bias, T, E, k, renorm, ids, gates, hdr, nullptr, 1, 0,
                             R, max_ranks);
  const TileGeom geom = layout_tiles(T);
  return launch_any<true>(env, logits, bias, T, E, k, renorm, ids, gates, hdr, tables, geom.TT,
                          half_words, R, max_ranks);
}

}  // namespace moe
