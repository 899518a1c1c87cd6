// dispatch.cu -- step 4: permute/scatter token rows into the layout.
//
// "GPU MoE all-to-all" (aicassindra), section "Bucketing: cut the message
// count, not the byte count": the permutation is fused into the kernel that
// stages the rows, so each token row is read once and written k times; and
// section "Latency-bound at decode, bandwidth-bound at prefill": the optional
// lower-precision (e4m3) copy, since the rows feed a matmul that would cast
// them anyway.
//
// Token-major and HBM-bound: no step is a contraction, so the kernel is a
// streaming copy.  Each warp loads a 32*CPT-chunk slice of one token row once
// (16-byte L1-bypassing loads) and issues k 16-byte stores per chunk.  Grid:
// the CTAs that fit on the GPU at once, striding over (token, slice) tasks.
//
// FP8 variant: per 128-channel block, amax by xor shuffle, scale = amax/448,
// inv = 448/amax (IEEE division), codes = cvt.rn.satfinite.e4m3x2(x * inv),
// 8-byte stores.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "bulk.cuh"
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 256;

// One warp per (token, slice of 32*CPT chunks): lane l holds chunks
// slice*32*CPT + l + 32*i, so each warp load or store is one contiguous 512 B
// run.  Lane j < k fetches dst_pos[t][j] once; the rows are broadcast by shuffle.
// x_ready (the fused steps 1-4, behind this library's layout kernel): x is
// complete, so the first task's rows are loaded before waiting for dst_pos.
template <int CPT>
__global__ void __launch_bounds__(kThreads)
    dispatch_bf16_kernel(const char* __restrict__ x, const int32_t* __restrict__ dst_pos, int T,
                         int H, int k, int64_t N, char* __restrict__ out, WsHeader* hdr,
                         int x_ready) {
  const int lane = threadIdx.x & 31;
  const int C8 = H >> 3;  // 16-byte chunks per row
  const int S = (C8 + 32 * CPT - 1) / (32 * CPT);
  const int64_t tasks = (int64_t)T * S;
  const size_t row_bytes = (size_t)H * 2;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
  const int64_t task0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  auto load_rows = [&](int64_t task, uint4 (&v)[CPT]) {
    const int t = (int)((uint32_t)task / (uint32_t)S);  // tasks < 2^31 (host check)
    const int cb = (int)((uint32_t)task - (uint32_t)t * (uint32_t)S) * 32 * CPT + lane;
    const char* src = x + (size_t)t * row_bytes;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = cb + 32 * i;
      if (c < C8) v[i] = ld16_stream(src + (size_t)c * 16);
    }
  };
  uint4 v0[CPT];
  if (x_ready && task0 < tasks) load_rows(task0, v0);
  pdl_wait();  // dst_pos (and, unless x_ready, x) may come from the kernel launched just before
  pdl_trigger();
  for (int64_t task = task0; task < tasks; task += nw) {
    const int t = (int)((uint32_t)task / (uint32_t)S);
    const int cb = (int)((uint32_t)task - (uint32_t)t * (uint32_t)S) * 32 * CPT + lane;
    uint4 v[CPT];
    if (x_ready && task == task0) {
#pragma unroll
      for (int i = 0; i < CPT; ++i) v[i] = v0[i];
    } else {
      load_rows(task, v);
    }
    const int pl = lane < k ? __ldg(dst_pos + (size_t)t * k + lane) : -1;
    for (int j = 0; j < k; ++j) {
      const int p = __shfl_sync(kFull, pl, j);
      if (p < 0) continue;
      if (p >= N) {
        if (lane == 0) report(hdr, MOE_ERR_DEVICE_RANGE, p);
        continue;
      }
      char* dst = out + (size_t)p * row_bytes;
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = cb + 32 * i;
        if (c < C8) st16(dst + (size_t)c * 16, v[i]);
      }
    }
  }
}

// Bulk-copy (TMA) variant for rows of 1-32 KiB.  Each CTA runs kBulkWarps
// independent pipelines over units (a token row, or a slice of one when there
// are too few tokens to keep every SM busy); lane 0 of a warp streams its
// units through `stages` shared-memory buffers: a bulk load global -> shared
// completes on the stage's mbarrier, then k bulk stores shared -> global (one
// bulk group per unit) write the copies, and the stage is refilled once the
// previous unit's group has finished reading it.  No thread touches the row
// data, so the LSU carries only the dst_pos loads.  Every wait is bounded.
constexpr int kBulkWarps = 4;
constexpr int kBulkMaxStages = 8;
constexpr uint64_t kBulkTimeoutNs = 1000000000ull;

__global__ void __launch_bounds__(kBulkWarps * 32)
    dispatch_bf16_bulk_kernel(const char* __restrict__ x, const int32_t* __restrict__ dst_pos,
                              int T, int H, int k, int64_t N, char* __restrict__ out, int stages,
                              uint32_t stage_bytes, int nsl, uint32_t slice_bytes, int x_ready,
                              int evict_first, WsHeader* hdr) {
  extern __shared__ __align__(128) unsigned char sbuf[];
  __shared__ uint64_t bars[kBulkWarps][kBulkMaxStages];
  // x_ready: the kernel launched just before this one did not write x, and
  // every kernel before it has finished (true behind this library's own route
  // and layout kernels, which each wait for their predecessor before letting
  // the next start), so the first rows can be fetched before the wait below.
  if (!x_ready) {
    pdl_wait();  // x and dst_pos may come from the kernel launched just before
    pdl_trigger();
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row = (size_t)H * 2;
  unsigned char* st = sbuf + (size_t)w * stages * stage_bytes;
  uint64_t* bar = bars[w];
  if (lane == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&bar[s], 1);
    mbar_fence_init();
  }
  __syncwarp();
  const int64_t units = (int64_t)T * nsl;
  const int64_t stride = (int64_t)gridDim.x * kBulkWarps;
  const int64_t first = (int64_t)blockIdx.x * kBulkWarps + w;
  const int64_t count = first < units ? (units - 1 - first) / stride + 1 : 0;
  // unit -> token, byte offset in the row, bytes
  // units < 2^31 (T * H/8 < 2^31 is checked on the host)
  auto unit_tok = [&](int64_t i) { return (uint32_t)(first + i * stride) / (uint32_t)nsl; };
  auto unit_off = [&](int64_t i) {
    return ((uint32_t)(first + i * stride) % (uint32_t)nsl) * slice_bytes;
  };
  auto unit_len = [&](int64_t i) {
    const uint32_t o = unit_off(i);
    return (uint32_t)min((size_t)slice_bytes, row - o);
  };
  auto issue_load = [&](int64_t i) {
    const int sn = (int)(i % stages);
    const uint32_t len = unit_len(i);
    mbar_arrive_expect_tx(&bar[sn], len);
    bulk_load(st + (size_t)sn * stage_bytes, x + (size_t)unit_tok(i) * row + unit_off(i), len,
              &bar[sn]);
  };
  int64_t issued = 0;  // loads issued (lane 0)
  if (lane == 0)
    for (; issued < count && issued < stages - 1; ++issued) issue_load(issued);
  if (x_ready) {  // dst_pos comes from the kernel launched just before
    pdl_wait();
    pdl_trigger();
  }
  uint32_t parity = 0;  // bit s: the phase stage s completes next
  bool ok = true;
  const uint64_t pol = l2_evict_first_policy();
  int pl = (count > 0 && lane < k) ? __ldg(dst_pos + (size_t)unit_tok(0) * k + lane) : -1;
  for (int64_t i = 0; i < count && ok; ++i) {
    const int s = (int)(i % stages);
    const int p_cur = pl;
    if (i + 1 < count && lane < k)  // next unit's rows, while this one streams
      pl = __ldg(dst_pos + (size_t)unit_tok(i + 1) * k + lane);
    if (lane == 0) {
      ok = mbar_wait_bounded(&bar[s], (parity >> s) & 1u, kBulkTimeoutNs);
      parity ^= 1u << s;
      if (!ok) report(hdr, MOE_ERR_DEVICE_TIMEOUT, (int)unit_tok(i));
    }
    ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    if (!ok) break;
    const uint32_t off = unit_off(i), len = unit_len(i);
    for (int j = 0; j < k; ++j) {
      const int p = __shfl_sync(kFull, p_cur, j);
      if (lane == 0 && p >= 0) {
        if (p < N)
          if (evict_first)  // output larger than L2: let its lines go back to DRAM early
            bulk_store_hint(out + (size_t)p * row + off, st + (size_t)s * stage_bytes, len, pol);
          else
            bulk_store(out + (size_t)p * row + off, st + (size_t)s * stage_bytes, len);
        else
          report(hdr, MOE_ERR_DEVICE_RANGE, p);
      }
    }
    if (lane == 0) {
      bulk_commit();
      if (issued < count) {  // refill the stage unit i-1 used
        bulk_wait_read<1>();
        issue_load(issued);
        ++issued;
      }
    }
    __syncwarp();
  }
  if (lane == 0) {
    bulk_wait_all();
    if (!ok) {  // let the loads still in flight land before the CTA exits
      for (int s = 0; s < stages; ++s)
        (void)mbar_wait_bounded(&bar[s], (parity >> s) & 1u, kBulkTimeoutNs);
    }
  }
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

// Same warp-per-(token, slice) mapping; the 16 chunks of a 128-channel
// block are 16 aligned lanes (slices start at multiples of 32 chunks), so the
// block's amax is a 4-step xor shuffle inside each half-warp.
template <int CPT>
__global__ void __launch_bounds__(kThreads)
    dispatch_fp8_kernel(const char* __restrict__ x, const int32_t* __restrict__ dst_pos, int T,
                        int H, int k, int64_t N, uint8_t* __restrict__ out,
                        float* __restrict__ scales, WsHeader* hdr) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int C8 = H >> 3;
  const int S = (C8 + 32 * CPT - 1) / (32 * CPT);
  const int nb = H >> 7;  // scale blocks per row
  const int64_t tasks = (int64_t)T * S;
  const size_t row_bytes = (size_t)H * 2;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
  for (int64_t task = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5; task < tasks;
       task += nw) {
    const int t = (int)((uint32_t)task / (uint32_t)S);  // tasks < 2^31 (host check)
    const int cb = (int)((uint32_t)task - (uint32_t)t * (uint32_t)S) * 32 * CPT + lane;
    const char* src = x + (size_t)t * row_bytes;
    uint32_t q[CPT][2];
    float s[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = cb + 32 * i;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (c < C8) v = ld16_stream(src + (size_t)c * 16);
      float f[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                    bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
      if (amax > 0.0f) {
        const float inv = __fdiv_rn(448.0f, amax);
        s[i] = __fdiv_rn(amax, 448.0f);
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(f[e], inv);
        q[i][0] = pack_e4m3x4(f[0], f[1], f[2], f[3]);
        q[i][1] = pack_e4m3x4(f[4], f[5], f[6], f[7]);
      } else {
        s[i] = 0.0f;
        q[i][0] = 0u;
        q[i][1] = 0u;
      }
    }
    const int pl = lane < k ? __ldg(dst_pos + (size_t)t * k + lane) : -1;
    for (int j = 0; j < k; ++j) {
      const int p = __shfl_sync(kFull, pl, j);
      if (p < 0) continue;
      if (p >= N) {
        if (lane == 0) report(hdr, MOE_ERR_DEVICE_RANGE, p);
        continue;
      }
      uint8_t* dst = out + (size_t)p * H;
      float* sdst = scales + (size_t)p * nb;
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = cb + 32 * i;
        if (c < C8) {
          *reinterpret_cast<uint2*>(dst + (size_t)c * 8) = make_uint2(q[i][0], q[i][1]);
          if ((c & 15) == 0) sdst[c >> 4] = s[i];
        }
      }
    }
  }
}

// FP8 with bulk stores, for H a multiple of 512 and rows of at most 8 KiB of
// codes: each warp streams its tokens; lane l quantises channels
// 512g + 16l .. +16 of every 512-channel group g (a 128-channel block is 8
// aligned lanes, its amax a 3-step xor shuffle), writes the codes and scales
// into one of kFp8Stages shared-memory stages; lane 0 issues the k bulk
// stores of the codes row (one bulk group per token) and the lanes write the
// k copies of the scales row with ordinary coalesced stores.  The first
// kFp8PrefetchGroups groups of the warp's next token are loaded into
// registers as soon as this token is quantised, so their latency hides
// behind this token's stores and the wait for a free stage.
constexpr int kFp8Stages = 4;
constexpr int kFp8PrefetchGroups = 4;

__global__ void __launch_bounds__(kBulkWarps * 32)
    dispatch_fp8_bulk_kernel(const char* __restrict__ x, const int32_t* __restrict__ dst_pos,
                             int T, int H, int k, int64_t N, uint8_t* __restrict__ out,
                             float* __restrict__ scales, uint32_t stage_bytes, int evict_first,
                             WsHeader* hdr) {
  extern __shared__ __align__(128) unsigned char sbuf[];
  pdl_wait();  // x and dst_pos may come from the kernel launched just before
  pdl_trigger();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t pol = l2_evict_first_policy();
  unsigned char* st = sbuf + (size_t)w * kFp8Stages * stage_bytes;
  const int groups = H >> 9;  // 512-channel groups
  const size_t xrow = (size_t)H * 2;
  const int64_t stride = (int64_t)gridDim.x * kBulkWarps;
  int64_t t = (int64_t)blockIdx.x * kBulkWarps + w;
  int pl = (t < T && lane < k) ? __ldg(dst_pos + (size_t)t * k + lane) : -1;
  // the first groups of token tt, 32 bytes a lane each
  const int pf = groups < kFp8PrefetchGroups ? groups : kFp8PrefetchGroups;
  uint4 nx[2 * kFp8PrefetchGroups];
  auto prefetch = [&](int64_t tt) {
    const char* src = x + (size_t)tt * xrow;
#pragma unroll
    for (int g = 0; g < kFp8PrefetchGroups; ++g) {
      const int ch = 512 * g + 16 * lane;
      if (tt < T && g < pf) {
        nx[2 * g] = ld16_stream(src + (size_t)ch * 2);
        nx[2 * g + 1] = ld16_stream(src + (size_t)ch * 2 + 16);
      }
    }
  };
  prefetch(t);
  for (int64_t i = 0; t < T; ++i, t += stride) {
    const int s = (int)(i % kFp8Stages);
    unsigned char* sp = st + (size_t)s * stage_bytes;
    const int p_cur = pl;
    if (t + stride < T && lane < k) pl = __ldg(dst_pos + (size_t)(t + stride) * k + lane);
    // the stores issued from this stage kFp8Stages tokens ago have read it
    if (lane == 0) bulk_wait_read<kFp8Stages - 1>();
    __syncwarp();
    const char* src = x + (size_t)t * xrow;
    auto quantise = [&](int g, const uint4& v0, const uint4& v1) {
      const int ch = 512 * g + 16 * lane;
      float f[16] = {bf16lo(v0.x), bf16hi(v0.x), bf16lo(v0.y), bf16hi(v0.y),
                     bf16lo(v0.z), bf16hi(v0.z), bf16lo(v0.w), bf16hi(v0.w),
                     bf16lo(v1.x), bf16hi(v1.x), bf16lo(v1.y), bf16hi(v1.y),
                     bf16lo(v1.z), bf16hi(v1.z), bf16lo(v1.w), bf16hi(v1.w)};
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
      uint4 q = make_uint4(0, 0, 0, 0);
      float scale = 0.0f;
      if (amax > 0.0f) {
        const float inv = __fdiv_rn(448.0f, amax);
        scale = __fdiv_rn(amax, 448.0f);
#pragma unroll
        for (int e = 0; e < 16; ++e) f[e] = __fmul_rn(f[e], inv);
        q.x = pack_e4m3x4(f[0], f[1], f[2], f[3]);
        q.y = pack_e4m3x4(f[4], f[5], f[6], f[7]);
        q.z = pack_e4m3x4(f[8], f[9], f[10], f[11]);
        q.w = pack_e4m3x4(f[12], f[13], f[14], f[15]);
      }
      *reinterpret_cast<uint4*>(sp + ch) = q;
      if ((lane & 7) == 0) *reinterpret_cast<float*>(sp + H + 4 * (ch >> 7)) = scale;
    };
#pragma unroll
    for (int g = 0; g < kFp8PrefetchGroups; ++g)
      if (g < pf) quantise(g, nx[2 * g], nx[2 * g + 1]);
#pragma unroll 4
    for (int g = kFp8PrefetchGroups; g < groups; ++g) {
      const int ch = 512 * g + 16 * lane;
      quantise(g, ld16_stream(src + (size_t)ch * 2), ld16_stream(src + (size_t)ch * 2 + 16));
    }
    prefetch(t + stride);  // in flight while this token's rows are stored
    fence_proxy_async_smem();  // these shared-memory writes before the bulk stores
    __syncwarp();
    // the scales row (H/128 floats, at most 64) by plain coalesced stores: a
    // bulk copy per 64-byte row would cost the copy engine as much as a row
    // of codes
    const int nb = H >> 7;
    const float s0 = lane < nb ? *reinterpret_cast<const float*>(sp + H + 4 * lane) : 0.0f;
    const float s1 = lane + 32 < nb ? *reinterpret_cast<const float*>(sp + H + 4 * (lane + 32)) : 0.0f;
    for (int j = 0; j < k; ++j) {
      const int p = __shfl_sync(kFull, p_cur, j);
      if (p < 0) continue;
      if (p >= N) {
        if (lane == 0) report(hdr, MOE_ERR_DEVICE_RANGE, p);
        continue;
      }
      float* srow_p = scales + (size_t)p * nb;
      if (evict_first) {  // output larger than L2: its lines go back to DRAM early
        if (lane == 0) bulk_store_hint(out + (size_t)p * H, sp, (uint32_t)H, pol);
        if (lane < nb) st_f32_hint(srow_p + lane, s0, pol);
        if (lane + 32 < nb) st_f32_hint(srow_p + lane + 32, s1, pol);
      } else {
        if (lane == 0) bulk_store(out + (size_t)p * H, sp, (uint32_t)H);
        if (lane < nb) srow_p[lane] = s0;
        if (lane + 32 < nb) srow_p[lane + 32] = s1;
      }
    }
    if (lane == 0) bulk_commit();
  }
  if (lane == 0) bulk_wait_all();
}

template <typename K>
int grid_for(K kernel, const LaunchEnv& env, int64_t units) {
  int per_sm = 1;
  if (blocks_per_sm(reinterpret_cast<const void*>(kernel), kThreads, 0, &per_sm) != cudaSuccess)
    per_sm = 1;
  const int64_t need = (units + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)env.num_sms * per_sm;
  int64_t g = need < cap ? need : cap;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_dispatch_bf16(const LaunchEnv& env, const void* x, const int32_t* dst_pos,
                                 int T, int H, int k, int64_t N, void* out, WsHeader* hdr,
                                 bool x_ready) {
  if (T == 0) return cudaSuccess;
  const int C8 = H / 8;
  const char* xs = static_cast<const char*>(x);
  char* o = static_cast<char*>(out);
  const uint32_t row = (uint32_t)H * 2u;
  // The bulk pipeline pays off once each warp has several rows to stream;
  // up to ~1k tokens one load and k stores per lane and slice finish sooner.
  if (row >= 1024 && row <= 32768 && T >= 2048) {
    const int64_t warps = (int64_t)env.num_sms * kBulkWarps;  // one CTA per SM
    // slices of >= 1 KiB (16-byte multiples) when the tokens alone cannot
    // give every pipeline two units
    int64_t nsl = (2 * warps + T - 1) / T;
    const int64_t max_nsl = row / 1024;
    if (nsl > max_nsl) nsl = max_nsl;
    if (nsl < 1) nsl = 1;
    const uint32_t slice = (uint32_t)((((row + nsl - 1) / nsl) + 15) / 16 * 16);
    nsl = (row + slice - 1) / slice;
    const uint32_t stage_bytes = (slice + 127u) & ~127u;
    int stages = (int)((200u * 1024u) / (kBulkWarps * stage_bytes));
    if (stages > kBulkMaxStages) stages = kBulkMaxStages;
    if (stages >= 2) {
      const size_t smem = (size_t)kBulkWarps * stages * stage_bytes;
      int per_sm = 1;
      const cudaError_t err =
          blocks_per_sm(reinterpret_cast<const void*>(dispatch_bf16_bulk_kernel),
                        kBulkWarps * 32, smem, &per_sm);
      if (err != cudaSuccess) return err;
      int64_t grid = (int64_t)per_sm * env.num_sms;
      const int64_t need = ((int64_t)T * nsl + kBulkWarps - 1) / kBulkWarps;
      if (grid > need) grid = need;
      // an output several times the 126 MB L2 cannot stay there for the next
      // kernel anyway: mark its lines evict-first so they are written back
      // while this kernel runs rather than during the next one
      const int evict_first = ((int64_t)T * k * row > (int64_t)192 << 20) ? 1 : 0;
      return launch_pdl(env, dispatch_bf16_bulk_kernel, dim3((unsigned)grid),
                        dim3(kBulkWarps * 32), smem, xs, dst_pos, T, H, k, N, o, stages,
                        stage_bytes, (int)nsl, slice, x_ready ? 1 : 0, evict_first, hdr);
    }
  }
  if (C8 >= 256) {
    auto kern = dispatch_bf16_kernel<2>;
    const int grid = grid_for(kern, env, (int64_t)T * ((C8 + 63) / 64) * 32);
    return launch_pdl(env, kern, dim3(grid), dim3(kThreads), 0, xs, dst_pos, T, H, k, N, o, hdr,
                      x_ready ? 1 : 0);
  } else {
    auto kern = dispatch_bf16_kernel<1>;
    const int grid = grid_for(kern, env, (int64_t)T * ((C8 + 31) / 32) * 32);
    return launch_pdl(env, kern, dim3(grid), dim3(kThreads), 0, xs, dst_pos, T, H, k, N, o, hdr,
                      x_ready ? 1 : 0);
  }
}

cudaError_t launch_dispatch_fp8(const LaunchEnv& env, const void* x, const int32_t* dst_pos,
                                int T, int H, int k, int64_t N, void* out, float* scales,
                                WsHeader* hdr) {
  if (T == 0) return cudaSuccess;
  const int C8 = H / 8;
  // staged variant: 512-channel groups per lane mapping (H % 512 == 0), a
  // 16-byte aligned output for the row bulk stores, and at most 64 scales a row
  if ((H % 512) == 0 && H <= 8192 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0) {
    const uint32_t stage_bytes = (uint32_t)(((size_t)H + H / 32 + 127) / 128 * 128);
    const size_t smem = (size_t)kBulkWarps * kFp8Stages * stage_bytes;
    int per_sm = 1;
    const cudaError_t err = blocks_per_sm(reinterpret_cast<const void*>(dispatch_fp8_bulk_kernel),
                                          kBulkWarps * 32, smem, &per_sm);
    if (err != cudaSuccess) return err;
    int64_t grid = (int64_t)per_sm * env.num_sms;
    const int64_t need = ((int64_t)T + kBulkWarps - 1) / kBulkWarps;
    if (grid > need) grid = need;
    const int evict_first = ((int64_t)T * k * (H + H / 32) > (int64_t)192 << 20) ? 1 : 0;
    return launch_pdl(env, dispatch_fp8_bulk_kernel, dim3((unsigned)grid), dim3(kBulkWarps * 32),
                      smem, static_cast<const char*>(x), dst_pos, T, H, k, N,
                      static_cast<uint8_t*>(out), scales, stage_bytes, evict_first, hdr);
  }
  auto kern = dispatch_fp8_kernel<1>;
  const int grid = grid_for(kern, env, (int64_t)T * ((C8 + 31) / 32) * 32);
  return launch_pdl(env, kern, dim3(grid), dim3(kThreads), 0, static_cast<const char*>(x), dst_pos,
                    T, H, k, N, static_cast<uint8_t*>(out), scales, hdr);
}

}  // namespace moe
