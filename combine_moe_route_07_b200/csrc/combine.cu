// combine.cu -- step 5: inverse-permutation gather, gate-weighted sum,
// shared-expert and residual add.
//
// "GPU MoE all-to-all" (aicassindra), section "Two collectives per layer, and
// what each one moves": k partial results come back along the inverse
// permutation and are scaled by the router's gate weights.  "MoE All-to-All
// Dispatch and Ragged Routing", section "Returning Tokens to the Original
// GPU": the residual x + dx is formed where x lives.  "19. All-to-all",
// section "Why the router can ruin your day": a dropped slot counts as if the
// token skipped that expert.
//
// Token-major gather, HBM-bound.  Every variant accumulates in fp32 in slot
// order j = 0..k-1 with round-to-nearest fused multiply-adds, adds the
// shared-expert row and then the residual row, and rounds to bf16 once, so all
// of them give the same bits.
//
// Register variant: each warp owns a 32*CPT-chunk slice of one token row; each
// lane issues the 16-byte loads of up to KB slots before using any of them.
// Bulk variant (dense layouts with many row slices per warp): the row slices
// arrive in shared memory by bulk copy (TMA), several tokens ahead of the
// arithmetic, so the bytes in flight do not cost registers.  Staged variant
// (dense layouts with rows wider than 8 KiB): one ring per CTA, a producer
// warp bringing in slices of several KiB per slot, eight consumer warps.
#include <cuda_bf16.h>

#include "bulk.cuh"
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 256;


__device__ __forceinline__ void fma8(float (&acc)[8], float g, const uint4& v) {
  acc[0] = __fmaf_rn(g, bf16lo(v.x), acc[0]);
  acc[1] = __fmaf_rn(g, bf16hi(v.x), acc[1]);
  acc[2] = __fmaf_rn(g, bf16lo(v.y), acc[2]);
  acc[3] = __fmaf_rn(g, bf16hi(v.y), acc[3]);
  acc[4] = __fmaf_rn(g, bf16lo(v.z), acc[4]);
  acc[5] = __fmaf_rn(g, bf16hi(v.z), acc[5]);
  acc[6] = __fmaf_rn(g, bf16lo(v.w), acc[6]);
  acc[7] = __fmaf_rn(g, bf16hi(v.w), acc[7]);
}

__device__ __forceinline__ void add8(float (&acc)[8], const uint4& v) {
  acc[0] = __fadd_rn(acc[0], bf16lo(v.x));
  acc[1] = __fadd_rn(acc[1], bf16hi(v.x));
  acc[2] = __fadd_rn(acc[2], bf16lo(v.y));
  acc[3] = __fadd_rn(acc[3], bf16hi(v.y));
  acc[4] = __fadd_rn(acc[4], bf16lo(v.z));
  acc[5] = __fadd_rn(acc[5], bf16hi(v.z));
  acc[6] = __fadd_rn(acc[6], bf16lo(v.w));
  acc[7] = __fadd_rn(acc[7], bf16hi(v.w));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Two fp32 fused multiply-adds in one instruction (sm_100): acc[i] = g * x[i]
// + acc[i], each rounded to nearest like __fmaf_rn.
__device__ __forceinline__ void fma8_x2(float (&acc)[8], float g, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint64_t gg;
  asm("mov.b64 %0, {%1, %1};" : "=l"(gg) : "f"(g));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint64_t a, x, d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(acc[2 * i]), "f"(acc[2 * i + 1]));
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(w[i] << 16), "r"(w[i] & 0xffff0000u));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(gg), "l"(x), "l"(a));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(acc[2 * i]), "=f"(acc[2 * i + 1]) : "l"(d));
  }
}

// One warp per (token, slice of 32*CPT chunks); lane j < k fetches the row
// and gate of slot j once and the warp broadcasts them by shuffle.  With
// PF the next task's token, rows and gates are fetched while this one
// computes.  KB == 1 walks only the kept slots (capacity mode drops most
// slots of a skewed batch), a token with no kept slot and no shared or
// residual row just stores zeros; KB > 1 keeps KB slots' loads in flight
// and skips a batch whose slots are all dropped.
template <int CPT, int KB, int MINB, bool PF>
__global__ void __launch_bounds__(kThreads, MINB)
    combine_kernel(const char* __restrict__ y, const int32_t* __restrict__ dst_pos,
                   const float* __restrict__ gates, const char* __restrict__ shared,
                   const char* __restrict__ residual, int T, int H, int k, int64_t N,
                   char* __restrict__ out, WsHeader* hdr) {
  pdl_wait();  // y, gates and dst_pos may come from the kernel launched just before
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int C8 = H >> 3;
  const int S = (C8 + 32 * CPT - 1) / (32 * CPT);
  const int64_t tasks = (int64_t)T * S;
  const size_t row_bytes = (size_t)H * 2;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
  // token of task `task` and slot j of it (lane j < k), -1 when dropped or
  // out of range
  auto fetch = [&](int64_t task, int& t, int& p, float& g) {
    t = task < tasks ? (int)((uint32_t)task / (uint32_t)S) : 0;  // tasks < 2^31 (host check)
    p = -1;
    g = 0.0f;
    if (task < tasks && lane < k) {
      p = __ldg(dst_pos + (size_t)t * k + lane);
      g = __ldg(gates + (size_t)t * k + lane);
      if (p >= N) {
        report(hdr, MOE_ERR_DEVICE_RANGE, p);
        p = -1;
      }
    }
  };
  int64_t task = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  int tl, pl, tn = 0, pn = -1;
  float gl, gn = 0.0f;
  fetch(task, tl, pl, gl);
  for (; task < tasks; task += nw) {
    if (PF) fetch(task + nw, tn, pn, gn);
    const int t = PF ? tl : (int)((uint32_t)task / (uint32_t)S);
    const int cb = (int)((uint32_t)task - (uint32_t)t * (uint32_t)S) * 32 * CPT + lane;
    const unsigned kept = __ballot_sync(kFull, pl >= 0);
    if (KB == 1 && kept == 0u && shared == nullptr && residual == nullptr) {
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = cb + 32 * i;
        if (c < C8) st16(out + (size_t)t * row_bytes + (size_t)c * 16, make_uint4(0, 0, 0, 0));
      }
    } else {
      float acc[CPT][8];
#pragma unroll
      for (int i = 0; i < CPT; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.0f;

      if constexpr (KB == 1) {
        for (unsigned m = kept; m != 0u; m &= m - 1u) {  // kept slots, ascending
          const int j = __ffs(m) - 1;
          const int p = __shfl_sync(kFull, pl, j);
          const float g = __shfl_sync(kFull, gl, j);
          const char* src = y + (size_t)p * row_bytes;
          uint4 v[CPT];
#pragma unroll
          for (int i = 0; i < CPT; ++i) {
            const int c = cb + 32 * i;
            v[i] = c < C8 ? ld16_stream(src + (size_t)c * 16) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int i = 0; i < CPT; ++i) fma8(acc[i], g, v[i]);
        }
      } else {
        for (int j0 = 0; j0 < k; j0 += KB) {
          if (((kept >> j0) & ((1u << KB) - 1u)) == 0u) continue;  // every slot dropped
          uint4 v[KB][CPT];
          float gw[KB];
          int pp[KB];
#pragma unroll
          for (int jj = 0; jj < KB; ++jj) {
            const int j = j0 + jj;  // j < 32: the shuffle source is always a lane
            pp[jj] = __shfl_sync(kFull, pl, j & 31);
            gw[jj] = __shfl_sync(kFull, gl, j & 31);
            if (j >= k) pp[jj] = -1;
            const char* src = y + (size_t)(pp[jj] < 0 ? 0 : pp[jj]) * row_bytes;
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
              const int c = cb + 32 * i;
              if (pp[jj] >= 0 && c < C8)
                v[jj][i] = ld16_stream(src + (size_t)c * 16);
              else
                v[jj][i] = make_uint4(0, 0, 0, 0);
            }
          }
#pragma unroll
          for (int jj = 0; jj < KB; ++jj)
            if (pp[jj] >= 0) {
#pragma unroll
              for (int i = 0; i < CPT; ++i) fma8(acc[i], gw[jj], v[jj][i]);
            }
        }
      }

#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = cb + 32 * i;
        if (c >= C8) continue;
        const size_t off = (size_t)t * row_bytes + (size_t)c * 16;
        if (shared != nullptr) add8(acc[i], ld16_stream(shared + off));
        if (residual != nullptr) add8(acc[i], ld16_stream(residual + off));
        uint4 o;
        o.x = pack_bf16x2(acc[i][0], acc[i][1]);
        o.y = pack_bf16x2(acc[i][2], acc[i][3]);
        o.z = pack_bf16x2(acc[i][4], acc[i][5]);
        o.w = pack_bf16x2(acc[i][6], acc[i][7]);
        st16(out + off, o);
      }
    }
    if (PF) {
      tl = tn;
      pl = pn;
      gl = gn;
    } else {
      fetch(task + nw, tl, pl, gl);
    }
  }
}

// Bulk variant.  One CTA per SM of 24 warps (16 when the stages of k plus the
// shared and residual slots do not fit twice per warp for 24); warp w owns a contiguous
// range of units (token t, 512-byte slice s of the row), so consecutive units
// mostly share a token and its dst_pos/gates (fetched one token ahead).  Per
// warp, a ring of `ns` shared-memory stages each holds one unit: the kept
// slots' slices of y, then the shared-expert and residual slices.  Unit u+ns-1
// is issued (lanes j < k each start one bulk copy of slot j; lanes 0 and 1 the
// shared and residual slices) before the warp waits for unit u, so ns-1 units
// are in flight while it computes.  Lane l computes the 16-byte chunk l of the
// slice.  Waits are bounded: a stage that does not fill within a second sets
// MOE_ERR_DEVICE_TIMEOUT, and the warp waits (bounded) for its copies still in
// flight before it exits.
constexpr int kBulkMaxWarps = 24;
constexpr int kBulkMinWarps = 16;
constexpr int kBulkMaxStages = 8;
constexpr uint32_t kBulkSlice = 512;
constexpr size_t kBulkSmemBudget = 200u * 1024u;
constexpr uint64_t kBulkTimeoutNs = 1000000000ull;

template <int KMAX>
__global__ void __launch_bounds__(kBulkMaxWarps * 32, 1)
    combine_bulk_kernel(const char* __restrict__ y, const int32_t* __restrict__ dst_pos,
                        const float* __restrict__ gates, const char* __restrict__ shared,
                        const char* __restrict__ residual, int T, int H, int k, int64_t N,
                        char* __restrict__ out, WsHeader* hdr, int ns, uint32_t stage_bytes) {
  extern __shared__ __align__(128) unsigned char sbuf[];
  __shared__ uint64_t bars[kBulkMaxWarps][kBulkMaxStages];
  __shared__ float sgate[kBulkMaxWarps][kBulkMaxStages][32];  // gate of each slot, per stage
  __shared__ uint32_t skept[kBulkMaxWarps][kBulkMaxStages];   // kept-slot mask, per stage
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t row = (uint32_t)H * 2;
  const int nsl = (int)((row + kBulkSlice - 1) / kBulkSlice);
  const int extra = (shared != nullptr) + (residual != nullptr);
  unsigned char* ring = sbuf + (size_t)w * ns * stage_bytes;
  uint64_t* bar = bars[w];
  if (lane == 0) {
    for (int s = 0; s < ns; ++s) mbar_init(&bar[s], 1);
    mbar_fence_init();
  }
  __syncwarp();
  pdl_wait();  // y, gates and dst_pos may come from the kernel launched just before
  pdl_trigger();
  const int64_t units = (int64_t)T * nsl;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + w;
  const int64_t u0 = units * wid / nwarps, u1 = units * (wid + 1) / nwarps;
  if (u0 >= u1) return;
  const int nunits = (int)(u1 - u0);
  const int t0 = (int)(u0 / nsl), sl0 = (int)(u0 - (int64_t)t0 * nsl);

  // issue side: token it, slice isl, stage is; slots of token it (ip, ig)
  // and of token it+1 (np, ng, checked when they are used)
  int it = t0, isl = sl0, is = 0;
  int ip = -1, np = -1;
  float ig = 0.0f, ng = 0.0f;
  if (lane < k) {
    ip = __ldg(dst_pos + (size_t)t0 * k + lane);
    ig = __ldg(gates + (size_t)t0 * k + lane);
    if (t0 + 1 < T) {
      np = __ldg(dst_pos + (size_t)(t0 + 1) * k + lane);
      ng = __ldg(gates + (size_t)(t0 + 1) * k + lane);
    }
  }
  if (ip >= N) {
    report(hdr, MOE_ERR_DEVICE_RANGE, ip);
    ip = -1;
  }
  auto issue = [&]() {
    const uint32_t off = (uint32_t)isl * kBulkSlice;
    const uint32_t len = min(kBulkSlice, row - off);
    const unsigned kept = __ballot_sync(kFull, ip >= 0);
    sgate[w][is][lane] = ig;
    if (lane == 0) {
      skept[w][is] = kept;
      mbar_arrive_expect_tx(&bar[is], ((uint32_t)__popc(kept) + (uint32_t)extra) * len);
    }
    __syncwarp();
    unsigned char* sp = ring + (size_t)is * stage_bytes;
    if (ip >= 0) bulk_load(sp + (size_t)lane * kBulkSlice, y + (size_t)ip * row + off, len, &bar[is]);
    if (lane == 0 && shared != nullptr)
      bulk_load(sp + (size_t)k * kBulkSlice, shared + (size_t)it * row + off, len, &bar[is]);
    if (lane == 1 && residual != nullptr)
      bulk_load(sp + (size_t)(k + extra - 1) * kBulkSlice, residual + (size_t)it * row + off, len,
                &bar[is]);
    if (++is == ns) is = 0;
    if (++isl == nsl) {
      isl = 0;
      ++it;
      ip = np;
      ig = ng;
      if (ip >= N) {
        report(hdr, MOE_ERR_DEVICE_RANGE, ip);
        ip = -1;
      }
      np = -1;
      ng = 0.0f;
      if (it + 1 < T && lane < k) {
        np = __ldg(dst_pos + (size_t)(it + 1) * k + lane);
        ng = __ldg(gates + (size_t)(it + 1) * k + lane);
      }
    }
  };

  int issued = 0;
  for (; issued < nunits && issued < ns - 1; ++issued) issue();
  int ct = t0, csl = sl0, cs = 0;
  uint32_t parity = 0;  // bit s: phase parity stage s waits for next
  for (int u = 0; u < nunits; ++u) {
    // the stage of unit u-1 is free again: refill it with unit u+ns-1
    if (issued < nunits) {
      issue();
      ++issued;
    }
    const bool ok = mbar_wait_bounded(&bar[cs], (parity >> cs) & 1u, kBulkTimeoutNs);
    if (!__all_sync(kFull, ok)) {
      if (lane == 0) report(hdr, MOE_ERR_DEVICE_TIMEOUT, ct);
      int s2 = cs;  // let the copies still in flight land before the warp exits
      for (int v = u; v < issued; ++v) {
        (void)mbar_wait_bounded(&bar[s2], (parity >> s2) & 1u, kBulkTimeoutNs);
        parity ^= 1u << s2;
        if (++s2 == ns) s2 = 0;
      }
      return;
    }
    parity ^= 1u << cs;
    const uint32_t off = (uint32_t)csl * kBulkSlice;
    const uint32_t len = min(kBulkSlice, row - off);
    if ((uint32_t)lane * 16 < len) {
      const unsigned kept = skept[w][cs];
      const unsigned char* sp = ring + (size_t)cs * stage_bytes + lane * 16;
      float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && ((kept >> j) & 1u))
          fma8_x2(acc, sgate[w][cs][j],
                  *reinterpret_cast<const uint4*>(sp + (size_t)j * kBulkSlice));
      if (shared != nullptr)
        add8(acc, *reinterpret_cast<const uint4*>(sp + (size_t)k * kBulkSlice));
      if (residual != nullptr)
        add8(acc, *reinterpret_cast<const uint4*>(sp + (size_t)(k + extra - 1) * kBulkSlice));
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      st16(out + (size_t)ct * row + off + lane * 16, o);
    }
    __syncwarp();  // every lane is done with stage cs before it is refilled
    if (++cs == ns) cs = 0;
    if (++csl == nsl) {
      csl = 0;
      ++ct;
    }
  }
}

// Staged variant: one ring of shared-memory stages per CTA, filled by one
// producer warp and read by kStageConsumers consumer warps.  A unit is a slice
// of SL bytes (a whole row, or an even part of it) of one token; its stage
// holds that slice of each kept slot's y row, then of the shared-expert row,
// then of the residual row, each brought in by ONE bulk copy of SL bytes
// (lane j of the producer copies slot j) -- bulk copies of a few KiB reach the
// DRAM read rate where 512-byte copies are bound by the copies' own cost.  The
// producer also leaves the unit's gates, kept-slot mask, token and slice in the
// stage's metadata before it arrives on the stage's "full" barrier; the
// consumer warps split the slice's 16-byte chunks, accumulate each in fp32 in
// slot order (fma.rn.f32x2), add the shared and residual rows, store the bf16
// result, and arrive on the stage's "empty" barrier.  Each CTA takes a
// contiguous range of units.  Every wait is bounded: a wait that gives up sets
// MOE_ERR_DEVICE_TIMEOUT and the abort flag, the producer stops issuing, and
// before it returns waits (bounded) for the copies of its last `ns` units, the
// only ones whose landing it has not already seen.
constexpr int kStageConsumers = 8;
constexpr int kStageThreads = (kStageConsumers + 1) * 32;
constexpr int kStageMax = 16;
constexpr int kStageMinRing = 3;    // stages the slice width is chosen for
constexpr size_t kStageSmemBudget = 200u * 1024u;

struct StageMeta {
  float gate[16];
  uint32_t kept;
  int token;
  uint32_t off;  // byte offset of the slice in the row
  uint32_t len;  // bytes of the slice
};

template <int KMAX>
__global__ void __launch_bounds__(kStageThreads, 1)
    combine_stage_kernel(const char* __restrict__ y, const int32_t* __restrict__ dst_pos,
                         const float* __restrict__ gates, const char* __restrict__ shared,
                         const char* __restrict__ residual, int T, int H, int k, int64_t N,
                         char* __restrict__ out, WsHeader* hdr, int ns, uint32_t SL, int nsl) {
  extern __shared__ __align__(128) unsigned char sbuf[];
  __shared__ uint64_t full[kStageMax], empty[kStageMax];
  __shared__ StageMeta meta[kStageMax];
  __shared__ volatile int abort_flag;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int extra = (shared != nullptr) + (residual != nullptr);
  const uint32_t row = (uint32_t)H * 2;
  const size_t stage_bytes = (size_t)(k + extra) * SL;
  if (threadIdx.x == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kStageConsumers);
    }
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  pdl_wait();  // y, gates and dst_pos may come from the kernel launched just before
  pdl_trigger();
  const int64_t units = (int64_t)T * nsl;
  const int64_t u0 = units * blockIdx.x / gridDim.x, u1 = units * (blockIdx.x + 1) / gridDim.x;
  const int n = (int)(u1 - u0);

  if (w == kStageConsumers) {  // the producer warp
    // slot `lane` of the current token (p, g) and of the next one (np, ng),
    // fetched one token ahead so their latency overlaps this token's copies
    auto fetch = [&](int t, int& pp, float& gg) {
      pp = -1;
      gg = 0.0f;
      if (t < T && lane < k) {
        pp = __ldg(dst_pos + (size_t)t * k + lane);
        gg = __ldg(gates + (size_t)t * k + lane);
      }
    };
    int cur_t = n > 0 ? (int)(u0 / nsl) : 0, p, np;
    float g, ng;
    fetch(cur_t, p, g);
    fetch(cur_t + 1, np, ng);
    if (p >= N) {
      report(hdr, MOE_ERR_DEVICE_RANGE, p);
      p = -1;
    }
    int issued = 0;
    for (int i = 0; i < n; ++i) {
      const int s = i % ns;
      if (i >= ns) {  // the consumers have finished with this stage's previous unit
        const bool ok = __all_sync(
            kFull, mbar_wait_bounded(&empty[s], (uint32_t)((i / ns) - 1) & 1u, kBulkTimeoutNs));
        if (!ok) {
          if (lane == 0) report(hdr, MOE_ERR_DEVICE_TIMEOUT, (int)(u0 + i));
          abort_flag = 1;
        }
      }
      if (__any_sync(kFull, abort_flag != 0)) break;  // one decision for the warp
      const int64_t u = u0 + i;
      const int t = (int)(u / nsl), sl = (int)(u - (int64_t)t * nsl);
      if (t != cur_t) {  // units are consecutive: t == cur_t + 1
        cur_t = t;
        p = np;
        g = ng;
        if (p >= N) {
          report(hdr, MOE_ERR_DEVICE_RANGE, p);
          p = -1;
        }
        fetch(t + 1, np, ng);
      }
      const uint32_t off = (uint32_t)sl * SL;
      const uint32_t len = min(SL, row - off);
      const unsigned kept = __ballot_sync(kFull, p >= 0);
      if (lane < KMAX) meta[s].gate[lane] = g;
      if (lane == 0) {
        meta[s].kept = kept;
        meta[s].token = t;
        meta[s].off = off;
        meta[s].len = len;
      }
      __syncwarp();
      if (lane == 0)  // after the metadata: the arrival releases it to the consumers
        mbar_arrive_expect_tx(&full[s], ((uint32_t)__popc(kept) + (uint32_t)extra) * len);
      __syncwarp();
      unsigned char* sp = sbuf + (size_t)s * stage_bytes;
      if (p >= 0) bulk_load(sp + (size_t)lane * SL, y + (size_t)p * row + off, len, &full[s]);
      if (lane == 0 && shared != nullptr)
        bulk_load(sp + (size_t)k * SL, shared + (size_t)t * row + off, len, &full[s]);
      if (lane == 1 && residual != nullptr)
        bulk_load(sp + (size_t)(k + extra - 1) * SL, residual + (size_t)t * row + off, len,
                  &full[s]);
      issued = i + 1;
    }
    if (lane == 0 && abort_flag) {  // the copies of the last ns units land before the CTA exits
      for (int i = issued > ns ? issued - ns : 0; i < issued; ++i)
        (void)mbar_wait_bounded(&full[i % ns], (uint32_t)(i / ns) & 1u, kBulkTimeoutNs);
    }
    return;
  }

  // the consumer warps: chunk c = (w*32 + lane) + kStageConsumers*32*r of the slice
  for (int i = 0; i < n; ++i) {
    const int s = i % ns;
    const bool ok =
        __all_sync(kFull, mbar_wait_bounded(&full[s], (uint32_t)(i / ns) & 1u, kBulkTimeoutNs));
    if (!ok) {
      if (lane == 0) report(hdr, MOE_ERR_DEVICE_TIMEOUT, (int)(u0 + i));
      abort_flag = 1;
    }
    if (__any_sync(kFull, abort_flag != 0)) return;  // one decision for the warp
    const StageMeta& m = meta[s];
    const unsigned kept = m.kept;
    const uint32_t len = m.len;
    const unsigned char* sp = sbuf + (size_t)s * stage_bytes;
    char* orow = out + (size_t)m.token * row + m.off;
    for (uint32_t c = (uint32_t)(w * 32 + lane) * 16; c < len; c += kStageConsumers * 32 * 16) {
      float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && ((kept >> j) & 1u))
          fma8_x2(acc, m.gate[j], *reinterpret_cast<const uint4*>(sp + (size_t)j * SL + c));
      if (shared != nullptr) add8(acc, *reinterpret_cast<const uint4*>(sp + (size_t)k * SL + c));
      if (residual != nullptr)
        add8(acc, *reinterpret_cast<const uint4*>(sp + (size_t)(k + extra - 1) * SL + c));
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      st16(orow + c, o);
    }
    __syncwarp();  // every lane is done with the stage
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

// Enough CTAs for one warp per task, at most the ones resident at once.
template <typename K>
int grid_for(K kernel, const LaunchEnv& env, int64_t tasks) {
  int per_sm = 1;
  if (blocks_per_sm(reinterpret_cast<const void*>(kernel), kThreads, 0, &per_sm) != cudaSuccess)
    per_sm = 1;
  const int64_t need = (tasks + kThreads / 32 - 1) / (kThreads / 32);
  const int64_t cap = (int64_t)env.num_sms * per_sm;
  int64_t g = need < cap ? need : cap;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_combine(const LaunchEnv& env, const void* y, const int32_t* dst_pos,
                           const float* gates, const void* shared, const void* residual, int T,
                           int H, int k, int64_t N, void* out, WsHeader* hdr, bool sparse) {
  if (T == 0) return cudaSuccess;
  const int C8 = H / 8;
  const char* ys = static_cast<const char*>(y);
  const char* sh = static_cast<const char*>(shared);
  const char* rs = static_cast<const char*>(residual);
  char* o = static_cast<char*>(out);
  const int extra = (shared != nullptr) + (residual != nullptr);
  // Dense layouts with rows wider than 8 KiB and at least 8 units per SM: the
  // staged variant, slices as wide as a ring of kStageMinRing stages allows
  // (whole rows, or the row cut evenly into 16-byte multiples).  On 14 KiB
  // rows its 7 KiB copies beat the bulk variant's 512-byte ones (Skewed
  // dropless combine 711 -> 650 us); on 8 KiB rows and narrower (Prefill,
  // Fine-grained) the bulk variant's 24 independent rings per SM do better.
  if ((size_t)H * 2 > 8192) {
    const size_t slots = (size_t)(k + extra);
    const size_t row = (size_t)H * 2;
    int64_t nsl = (int64_t)((slots * row * kStageMinRing + kStageSmemBudget - 1) / kStageSmemBudget);
    if (nsl < 1) nsl = 1;
    const uint32_t SL = (uint32_t)(((row + nsl - 1) / nsl + 15) / 16 * 16);
    nsl = (int64_t)((row + SL - 1) / SL);
    int ns = (int)(kStageSmemBudget / (slots * SL));
    if (ns > kStageMax) ns = kStageMax;
    if (!sparse && k <= 16 && ns >= 2 && (int64_t)T * nsl >= 8 * (int64_t)env.num_sms) {
      const size_t smem = (size_t)ns * slots * SL;
      auto kern = k <= 8 ? combine_stage_kernel<8> : combine_stage_kernel<16>;
      int per_sm = 1;
      const cudaError_t err =
          blocks_per_sm(reinterpret_cast<const void*>(kern), kStageThreads, smem, &per_sm);
      if (err != cudaSuccess) return err;
      int64_t grid = (int64_t)env.num_sms * per_sm;
      if (grid > (int64_t)T * nsl) grid = (int64_t)T * nsl;
      return launch_pdl(env, kern, dim3((unsigned)grid), dim3(kStageThreads), smem, ys, dst_pos,
                        gates, sh, rs, T, H, k, N, o, hdr, ns, SL, (int)nsl);
    }
  }
  // Dense layouts with at least 8 row slices per warp of a full bulk grid:
  // the bulk variant, when the stages of up to 12 slots (k plus the shared
  // and residual rows) fit twice per warp.  Warps matter more than ring
  // depth: 24 warps with two stages each tie or beat 16 with three, and wider
  // slices with fewer warps ran far slower.
  const uint32_t stage_bytes = (uint32_t)(k + extra) * kBulkSlice;
  const int W = kBulkSmemBudget / ((size_t)kBulkMaxWarps * stage_bytes) >= 2 ? kBulkMaxWarps
                                                                             : kBulkMinWarps;
  const int ns_fit = (int)(kBulkSmemBudget / ((size_t)W * stage_bytes));
  const int64_t slices = (int64_t)T * ((2 * (int64_t)H + kBulkSlice - 1) / kBulkSlice);
  if (!sparse && k <= 16 && ns_fit >= 2 && slices >= 8 * (int64_t)env.num_sms * W) {
    const int ns = ns_fit < kBulkMaxStages ? ns_fit : kBulkMaxStages;
    const size_t smem = (size_t)W * ns * stage_bytes;
    auto kern = k <= 8 ? combine_bulk_kernel<8> : combine_bulk_kernel<16>;
    int per_sm = 1;
    const cudaError_t err =
        blocks_per_sm(reinterpret_cast<const void*>(kern), W * 32, smem, &per_sm);
    if (err != cudaSuccess) return err;
    return launch_pdl(env, kern, dim3((unsigned)(env.num_sms * per_sm)), dim3(W * 32), smem, ys,
                      dst_pos, gates, sh, rs, T, H, k, N, o, hdr, ns, stage_bytes);
  }
  // Capacity mode drops most slots of a skewed batch: then each task moves
  // little and its latency dominates, so wider slices with the next task's
  // metadata prefetched win, one slot at a time (a slot's loads are skipped
  // alone when it is dropped, and nothing spills at 64 registers); dense
  // layouts do better with more warps, all k slots' loads in flight at once.
  if (sparse && C8 >= 128) {
    auto kern = combine_kernel<4, 1, 4, true>;
    const int grid = grid_for(kern, env, (int64_t)T * ((C8 + 127) / 128));
    return launch_pdl(env, kern, dim3(grid), dim3(kThreads), 0, ys, dst_pos, gates, sh, rs, T, H,
                      k, N, o, hdr);
  }
  auto kern = combine_kernel<1, 8, 4, false>;
  const int grid = grid_for(kern, env, (int64_t)T * ((C8 + 31) / 32));
  return launch_pdl(env, kern, dim3(grid), dim3(kThreads), 0, ys, dst_pos, gates, sh, rs, T, H, k,
                    N, o, hdr);
}

}  // namespace moe
