// route_core.cuh -- top-k selection and gates, one warp per token (or per
// group of tokens): the device side of step 1, used by route.cu.
//
// "19. All-to-all" (ai-from-scratch), section "Why the router can ruin your
// day": the per-expert balancing bias enters the top-k decision and nothing
// else; the mix weights come from the router's own scores.
//
// Lane l holds experts l, l+32, l+64, ... of each token in registers, as
// order-preserving 32-bit codes of key = logit + bias.  Each of the k rounds
// is two hardware warp reductions (redux.sync): the largest code, then the
// lowest expert id among the lanes holding it, which is the tie rule.  Four
// forms of the same selection: route_tokens (every code, k rounds; E <= 224),
// route_token_thr (a threshold first, then the few keys above it ranked
// against each other), route_token_smem (the threshold form with the row and
// the bias read from shared memory, only the codes in registers) and
// select_fast (the threshold form on the float keys of a staged row, which
// hands ties, NaN and large candidate sets to route_token_smem).  An optional
// rank limit clears the codes of all but the M best ranks first.  The gates
// are a softmax of the selected RAW logits evaluated in fp64 (k values per
// token): fp64 exponentials and sum, the quotient as the exponential times the
// correctly rounded fp64 reciprocal of the sum (a full fp64 division cost ~80
// more instructions per token), then one rounding to fp32.  That differs from
// rounding the exact fp64 quotient only when it lies within ~2^-52 of an fp32
// rounding boundary, far inside the 1e-6 gate tolerance.
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {

// Finite fp32 -> uint32 with the same order; -0 folds onto +0 first so the
// two compare equal.  No non-NaN key maps to 0, which marks "taken".
__device__ __forceinline__ uint32_t order_code(float f) {
  if (f == 0.0f) f = 0.0f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float an order code stands for (the inverse of order_code on codes of
// non-NaN floats; +0 for the code of a folded zero).
__device__ __forceinline__ float code_float(uint32_t c) {
  return __uint_as_float((c & 0x80000000u) ? (c & 0x7fffffffu) : ~c);
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

template <int NK>
__device__ __forceinline__ void load_bias(const float* bias, int E, int lane, float (&b)[NK]) {
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int e = lane + 32 * i;
    b[i] = (bias != nullptr && e < E) ? __ldg(bias + e) : 0.0f;
  }
}

// Rank limit: each token's experts come from at most M of the R ranks (expert
// e on rank e / (E/R)).  Group score of a rank = its largest key code; the M
// best ranks are kept (equal scores: the lower rank id), every other rank's
// codes are cleared to 0 ("taken") before the selection.  "19. All-to-all",
// opening section (each token limited to a few nodes); "GPU MoE all-to-all",
// section "The node boundary is the design decision".  `smem` is this warp's
// R + ceil(R/32) words (used only when E/R neither divides nor is a multiple
// of 32).  Off when M <= 0 or M >= R.
struct RankLimit {
  int R = 1;
  int M = 0;
  uint32_t* smem = nullptr;
  // per-lane constants, set once by init(): experts per rank, how ranks map
  // onto the lane-major keys, and this lane's place in that map
  int Er = 1;
  int mode = 0;  // 1: Er divides 32, R <= 64 (ranks inside a column); 2: whole columns; 0: other
  int step = 0;  // mode 1: ranks per column; mode 2: columns per rank
  int lane_rank = 0;
  bool lead = false;
  bool col_map = false;  // Er divides 32: key i of this lane is on rank i * step + lane_rank
  uint32_t magic = 0u;   // Er >= 2: ceil(2^32 / Er), n / Er == __umulhi(n, magic) for n < 2^16
  __device__ bool on() const { return M > 0 && M < R; }
  __device__ void init(int E, int lane) {
    Er = E / R;
    magic = Er >= 2 ? (uint32_t)((0x100000000ull + (uint64_t)Er - 1) / (uint64_t)Er) : 0u;
    col_map = Er <= 32 && (32 % Er) == 0;
    if (col_map) {
      step = 32 / Er;
      lane_rank = lane / Er;
      lead = (lane % Er) == 0;
    }
    if (col_map && R <= 64) {
      mode = 1;
    } else if ((Er & 31) == 0) {
      mode = 2;
      step = Er >> 5;
    } else {
      mode = 0;
    }
  }
};

template <int NK>
__device__ __forceinline__ void apply_rank_limit(uint32_t (&code)[NK], int E, int lane,
                                                 const RankLimit& L) {
  const int R = L.R;
  if (L.mode == 1) {
    // A rank is Er aligned lanes of one column (R <= 64): an xor-max over the
    // group gives the rank's score, the group's first lane stores it, and
    // lane l then holds the scores of ranks l and l+32; M rounds of a warp
    // arg-max (lower id on ties) fill a 64-bit mask of the kept ranks.
    uint32_t* rmax = L.smem;
#pragma unroll
    for (int i = 0; i < NK; ++i) {
      const bool valid = lane + 32 * i < E;
      uint32_t v = valid ? code[i] : 0u;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1)
        if (o < L.Er) v = max(v, __shfl_xor_sync(kFull, v, o));
      if (valid && L.lead) rmax[i * L.step + L.lane_rank] = v;
    }
    __syncwarp();
    const uint32_t s0 = lane < R ? rmax[lane] : 0u;
    const uint32_t s1 = lane + 32 < R ? rmax[lane + 32] : 0u;
    __syncwarp();  // the next token reuses the words
    uint64_t kept = 0ull;
    for (int m = 0; m < L.M; ++m) {
      const uint32_t b0 = ((kept >> lane) & 1ull) ? 0u : s0;  // valid scores are never 0
      const uint32_t b1 = ((kept >> (lane + 32)) & 1ull) ? 0u : s1;
      const uint32_t best = max(b0, b1);
      const uint32_t id = b0 >= b1 ? (uint32_t)lane : (uint32_t)(lane + 32);
      const uint32_t top = __reduce_max_sync(kFull, best);
      const uint32_t win = __reduce_min_sync(kFull, best == top ? id : 0xffffffffu);
      kept |= 1ull << win;
    }
#pragma unroll
    for (int i = 0; i < NK; ++i)
      if (((kept >> (i * L.step + L.lane_rank)) & 1ull) == 0ull) code[i] = 0u;
    return;
  }
  if (L.mode == 2) {
    // A rank is Er/32 whole columns: every lane ends up with every score
    // (R <= NK), so all lanes take the same M decisions without exchange.
    uint32_t sc[NK];  // sc[i]: score of the rank whose last column is i
    uint32_t acc = 0u;
#pragma unroll
    for (int i = 0; i < NK; ++i) {
      sc[i] = 0u;
      if (32 * i < E) {
        acc = max(acc, code[i]);
        if ((i + 1) % L.step == 0) {
          sc[i] = __reduce_max_sync(kFull, acc);
          acc = 0u;
        }
      }
    }
    uint32_t keep = 0u;  // bit i: the rank ending at column i is kept
    for (int m = 0; m < L.M; ++m) {
      uint32_t best = 0u;
      int bi = -1;
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if (32 * i < E && (i + 1) % L.step == 0 && ((keep >> i) & 1u) == 0u &&
            (bi < 0 || sc[i] > best)) {
          best = sc[i];
          bi = i;
        }
      keep |= 1u << bi;
    }
#pragma unroll
    for (int i = 0; i < NK; ++i) {  // column i belongs to the rank ending at its group's last column
      const int last = (i / L.step + 1) * L.step - 1;
      if (last >= NK || ((keep >> last) & 1u) == 0u) code[i] = 0u;
    }
    return;
  }
  // other sizes: shared-memory maxima and a shared bitmap of kept ranks
  uint32_t* rmax = L.smem;
  uint32_t* chosen = L.smem + R;
  for (int q = lane; q < (R + 31) / 32; q += 32) chosen[q] = 0u;
  for (int r = lane; r < R; r += 32) rmax[r] = 0u;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int e = lane + 32 * i;
    if (e < E && code[i] != 0u) atomicMax(&rmax[e / L.Er], code[i]);
  }
  __syncwarp();
  for (int m = 0; m < L.M; ++m) {
    uint32_t best = 0u;
    int bi = R;
    for (int r = lane; r < R; r += 32) {  // ascending r: strict > keeps the lower id
      if (((chosen[r >> 5] >> (r & 31)) & 1u) == 0u) {
        const uint32_t v = rmax[r];
        if (bi == R || v > best) {
          best = v;
          bi = r;
        }
      }
    }
    const uint32_t top = __reduce_max_sync(kFull, best);
    const uint32_t win =
        __reduce_min_sync(kFull, (bi < R && best == top) ? (uint32_t)bi : 0xffffffffu);
    if (lane == 0) chosen[win >> 5] |= 1u << (win & 31u);
    __syncwarp();
  }
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const int r = e / L.Er;
      if (((chosen[r >> 5] >> (r & 31)) & 1u) == 0u) code[i] = 0u;
    }
  }
  __syncwarp();  // the next token reuses the words
}

// Route tokens tok[0..TPW) (entries >= T are skipped).  On return lane j < k
// holds slot j of token u: expert sel_e[u], gate[u].  Returns the first token
// with a NaN key, or -1.
template <int NK, int TPW>
__device__ __forceinline__ int route_tokens(const float* __restrict__ logits, const int (&tok)[TPW],
                                            int T, const float (&b)[NK], int E, int k, int renorm,
                                            int lane, int (&sel_e)[TPW], float (&gate)[TPW],
                                            const RankLimit& lim = RankLimit()) {
  float raw[TPW][NK];
  uint32_t code[TPW][NK];
  int nan_tok = -1;
#pragma unroll
  for (int u = 0; u < TPW; ++u) {
    const bool live = tok[u] < T;
    const float* row = logits + (size_t)(live ? tok[u] : 0) * E;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < NK; ++i) {
      const int e = lane + 32 * i;
      if (live && e < E) {
        raw[u][i] = __ldcs(row + e);  // read once: streaming
        const float key = __fadd_rn(raw[u][i], b[i]);
        bad |= (key != key);
        code[u][i] = order_code(key);
      } else {
        raw[u][i] = -INFINITY;
        code[u][i] = 0u;
      }
    }
    if (__any_sync(kFull, bad) && nan_tok < 0) nan_tok = tok[u];
    if (lim.on()) apply_rank_limit<NK>(code[u], E, lane, lim);
  }

  float sel_raw[TPW];
#pragma unroll
  for (int u = 0; u < TPW; ++u) {
    sel_e[u] = 0;
    sel_raw[u] = 0.0f;
  }
  for (int j = 0; j < k; ++j) {
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
      uint32_t best = 0u;
      int bi = 0;
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if (code[u][i] > best) {  // strict: the lowest index wins ties
          best = code[u][i];
          bi = i;
        }
      const uint32_t top = __reduce_max_sync(kFull, best);
      const uint32_t cand = (best == top) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu;
      const uint32_t win = __reduce_min_sync(kFull, cand);
      float r = 0.0f;
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if ((uint32_t)(lane + 32 * i) == win) {
          code[u][i] = 0u;
          r = raw[u][i];
        }
      r = __shfl_sync(kFull, r, (int)(win & 31u));
      if (lane == j) {
        sel_e[u] = (int)win;
        sel_raw[u] = r;
      }
    }
  }

#pragma unroll
  for (int u = 0; u < TPW; ++u) {
    if (renorm) {
      const float m = warp_max_f(lane < k ? sel_raw[u] : -INFINITY);
      const double ex = (lane < k) ? exp((double)sel_raw[u] - (double)m) : 0.0;
      const double den = warp_sum_d(ex);
      gate[u] = (float)(ex * __drcp_rn(den));
    } else {
      float lm = -INFINITY;
#pragma unroll
      for (int i = 0; i < NK; ++i) lm = fmaxf(lm, raw[u][i]);
      const float m = warp_max_f(lm);
      double part = 0.0;
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if (lane + 32 * i < E) part += exp((double)raw[u][i] - (double)m);
      const double den = warp_sum_d(part);
      gate[u] = (float)(exp((double)sel_raw[u] - (double)m) * __drcp_rn(den));
    }
  }
  return nan_tok;
}


// Exact top-k through a threshold, for many keys per lane (NK >= 8).
// tau = the k-th largest of the 32 lane maxima: those k maxima are k distinct
// keys >= tau, so the k-th largest key is >= tau and no key below tau can be
// selected.  The warp compacts the keys >= tau (usually k to k+4 of them) into
// shared memory and ranks them (select_ranked).  More than kMaxCand candidates
// (heavy ties) falls back to route_tokens.  `cand` is this warp's 3*kMaxCand
// words of shared memory, 8-byte aligned.  (Rows staged in shared memory go
// through route_token_smem instead.)
constexpr int kMaxCand = 64;

// Slot order of `total` candidates: the key (code << 32) | ~id orders larger
// codes first and, among equal codes, lower ids first, and no two keys are
// equal, so candidate i's slot is the number of keys above its own.  Lanes i
// and i+32 rank candidates i and i+32 against every key (one broadcast load
// each), the candidates of slots j < k are scattered to slot j, and lane j < k
// returns slot j's expert (and, with RAW, its raw logit bits from `raw`).
// `key` holds kMaxCand keys and `raw` kMaxCand words; both are reused for the
// slots, and the warp is synchronised before they are written and on return.
template <bool RAW>
__device__ __forceinline__ void select_ranked(uint64_t* key, uint32_t* raw, int total, int k,
                                              int lane, int& sel_e, uint32_t& sel_raw) {
  const bool h0 = lane < total, h1 = lane + 32 < total;
  const uint64_t k0 = h0 ? key[lane] : 0ull;
  const uint64_t k1 = h1 ? key[lane + 32] : 0ull;
  uint32_t v0 = 0u, v1 = 0u;
  if (RAW) {
    v0 = h0 ? raw[lane] : 0u;
    v1 = h1 ? raw[lane + 32] : 0u;
  }
  int n0 = 0, n1 = 0;
  if (total <= 32) {
    for (int m = 0; m < total; ++m) n0 += key[m] > k0 ? 1 : 0;
  } else {
    for (int m = 0; m < total; ++m) {
      const uint64_t km = key[m];
      n0 += km > k0 ? 1 : 0;
      n1 += km > k1 ? 1 : 0;
    }
  }
  __syncwarp();  // every key has been read: the slots reuse the arrays
  uint32_t* slot_e = reinterpret_cast<uint32_t*>(key);
  if (h0 && n0 < k) {
    slot_e[n0] = ~(uint32_t)k0;
    if (RAW) raw[n0] = v0;
  }
  if (h1 && n1 < k) {
    slot_e[n1] = ~(uint32_t)k1;
    if (RAW) raw[n1] = v1;
  }
  __syncwarp();
  if (lane < k) {
    sel_e = (int)slot_e[lane];
    if (RAW) sel_raw = raw[lane];
  }
  __syncwarp();  // the next token may overwrite the arrays
}

template <int NK>
__device__ __forceinline__ int route_token_thr(const float* __restrict__ logits, int t, int T,
                                               const float (&b)[NK], int E, int k, int renorm,
                                               int lane, uint32_t* cand, int& sel_e,
                                               float& gate, const RankLimit& lim = RankLimit()) {
  float raw[NK];
  uint32_t code[NK];
  bool bad = false;
  const float* row = logits + (size_t)t * E;
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      raw[i] = __ldcs(row + e);
      const float key = __fadd_rn(raw[i], b[i]);
      bad |= (key != key);
      code[i] = order_code(key);
    } else {
      raw[i] = -INFINITY;
      code[i] = 0u;
    }
  }
  const int nan_tok = __any_sync(kFull, bad) ? t : -1;
  if (lim.on()) apply_rank_limit<NK>(code, E, lane, lim);

  // threshold: k-th largest lane maximum
  uint32_t mm = 0u;
#pragma unroll
  for (int i = 0; i < NK; ++i) mm = max(mm, code[i]);
  uint32_t tau = 0u;
  for (int j = 0; j < k; ++j) {
    const uint32_t top = __reduce_max_sync(kFull, mm);
    tau = top;
    const unsigned hold = __ballot_sync(kFull, mm == top);
    if (lane == __ffs(hold) - 1) mm = 0u;
  }
  int c = 0;
#pragma unroll
  for (int i = 0; i < NK; ++i) c += (code[i] != 0u && code[i] >= tau) ? 1 : 0;
  const int total = (int)__reduce_add_sync(kFull, (unsigned)c);
  if (total > kMaxCand) {  // heavy ties at the threshold: the full scan
    int tok[1] = {t}, e1[1];
    float g1[1];
    route_tokens<NK, 1>(logits, tok, T, b, E, k, renorm, lane, e1, g1, lim);
    sel_e = e1[0];
    gate = g1[0];
    return nan_tok;
  }
  int pre = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, pre, o);
    if (lane >= o) pre += y;
  }
  pre -= c;
  uint64_t* ckey = reinterpret_cast<uint64_t*>(cand);
  uint32_t* craw = cand + 2 * kMaxCand;
#pragma unroll
  for (int i = 0; i < NK; ++i)
    if (code[i] != 0u && code[i] >= tau) {
      ckey[pre] = ((uint64_t)code[i] << 32) | (uint64_t)(~(uint32_t)(lane + 32 * i));
      craw[pre] = __float_as_uint(raw[i]);
      ++pre;
    }
  __syncwarp();
  sel_e = 0;
  uint32_t rbits = 0u;
  select_ranked<true>(ckey, craw, total, k, lane, sel_e, rbits);
  const float sel_raw = __uint_as_float(rbits);

  if (renorm) {
    const float m = warp_max_f(lane < k ? sel_raw : -INFINITY);
    const double ex = (lane < k) ? exp((double)sel_raw - (double)m) : 0.0;
    const double den = warp_sum_d(ex);
    gate = (float)(ex * __drcp_rn(den));
  } else {
    float lm = -INFINITY;
#pragma unroll
    for (int i = 0; i < NK; ++i) lm = fmaxf(lm, raw[i]);
    const float m = warp_max_f(lm);
    double part = 0.0;
#pragma unroll
    for (int i = 0; i < NK; ++i)
      if (lane + 32 * i < E) part += exp((double)raw[i] - (double)m);
    const double den = warp_sum_d(part);
    gate = (float)(exp((double)sel_raw - (double)m) * __drcp_rn(den));
  }
  return nan_tok;
}

// Rank limit for a token whose row and bias sit in shared memory, decided
// before any key code is formed: lane l scores ranks l, l+32, ... straight
// from the row (the largest key code over the rank's experts) and M rounds of
// a warp arg-max pick the kept ranks.  R <= 64: returns the kept ranks as a
// 64-bit mask; larger R: marks them in this warp's shared bitmap (L.smem + R)
// and returns 0.
__device__ __forceinline__ uint64_t rank_limit_smem(const float* srow, const float* sbias,
                                                    int lane, const RankLimit& L) {
  const int R = L.R, Er = L.Er;
  auto score = [&](int r) {
    uint32_t best = 0u;
    for (int e = r * Er; e < (r + 1) * Er; ++e)
      best = max(best, order_code(__fadd_rn(srow[e], sbias[e])));
    return best;
  };
  if (R <= 64) {
    const uint32_t s0 = lane < R ? score(lane) : 0u;
    const uint32_t s1 = lane + 32 < R ? score(lane + 32) : 0u;
    uint64_t kept = 0ull;
    for (int m = 0; m < L.M; ++m) {
      const uint32_t b0 = ((kept >> lane) & 1ull) ? 0u : s0;  // valid scores are never 0
      const uint32_t b1 = ((kept >> (lane + 32)) & 1ull) ? 0u : s1;
      const uint32_t best = max(b0, b1);
      const uint32_t id = b0 >= b1 ? (uint32_t)lane : (uint32_t)(lane + 32);
      const uint32_t top = __reduce_max_sync(kFull, best);
      kept |= 1ull << __reduce_min_sync(kFull, best == top ? id : 0xffffffffu);
    }
    return kept;
  }
  uint32_t* rmax = L.smem;
  uint32_t* chosen = L.smem + R;
  __syncwarp();  // the previous token is done with the words
  for (int r = lane; r < R; r += 32) rmax[r] = score(r);
  for (int q = lane; q < (R + 31) / 32; q += 32) chosen[q] = 0u;
  __syncwarp();
  for (int m = 0; m < L.M; ++m) {
    uint32_t best = 0u;
    int bi = R;
    for (int r = lane; r < R; r += 32) {  // ascending r: strict > keeps the lower id
      if (((chosen[r >> 5] >> (r & 31)) & 1u) == 0u) {
        const uint32_t v = rmax[r];
        if (bi == R || v > best) {
          best = v;
          bi = r;
        }
      }
    }
    const uint32_t top = __reduce_max_sync(kFull, best);
    const uint32_t win =
        __reduce_min_sync(kFull, (bi < R && best == top) ? (uint32_t)bi : 0xffffffffu);
    if (lane == 0) chosen[win >> 5] |= 1u << (win & 31u);
    __syncwarp();
  }
  return 0ull;
}

// Is the rank of expert e kept?  (the mask or bitmap rank_limit_smem made)
__device__ __forceinline__ bool rank_kept(int e, int i, int lane, uint64_t kept,
                                          const RankLimit& L) {
  const int r = L.col_map ? i * L.step + L.lane_rank : (int)__umulhi((uint32_t)e, L.magic);
  if (L.R <= 64) return ((kept >> r) & 1ull) != 0ull;
  return ((L.smem[L.R + (r >> 5)] >> (r & 31)) & 1u) != 0u;
}

// Threshold top-k for a token whose logits row (and the bias) sit in shared
// memory: only the key codes live in registers, the raw logits are re-read
// from the row where they are needed (the candidates, the winner of a full
// scan, the full softmax without renorm).  The same decisions as
// route_token_thr: tau = the k-th largest lane maximum, compaction of the
// keys >= tau, k rounds over at most two candidates per lane; more than
// kMaxCand candidates (heavy ties) takes k rounds over all the codes.
template <int NK, bool LIMIT>
__device__ __forceinline__ int route_token_smem(const float* srow, const float* sbias, int t,
                                                int E, int k, int renorm, int lane,
                                                uint32_t* cand, int& sel_e, float& gate,
                                                const RankLimit& lim) {
  uint64_t kept = 0ull;
  if constexpr (LIMIT) kept = rank_limit_smem(srow, sbias, lane, lim);
  uint32_t code[NK];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const float key = __fadd_rn(srow[e], sbias[e]);
      bad |= (key != key);
      code[i] = order_code(key);
      if constexpr (LIMIT)
        if (!rank_kept(e, i, lane, kept, lim)) code[i] = 0u;
    } else {
      code[i] = 0u;
    }
  }
  const int nan_tok = __any_sync(kFull, bad) ? t : -1;

  uint32_t mm = 0u;
#pragma unroll
  for (int i = 0; i < NK; ++i) mm = max(mm, code[i]);
  uint32_t tau = 0u;
  for (int j = 0; j < k; ++j) {
    const uint32_t top = __reduce_max_sync(kFull, mm);
    tau = top;
    const unsigned hold = __ballot_sync(kFull, mm == top);
    if (lane == __ffs(hold) - 1) mm = 0u;
  }
  uint32_t cmask = 0u;  // bit i: key i of this lane is a candidate
#pragma unroll
  for (int i = 0; i < NK; ++i) cmask |= (code[i] != 0u && code[i] >= tau) ? (1u << i) : 0u;
  const int c = __popc(cmask);
  const int total = (int)__reduce_add_sync(kFull, (unsigned)c);

  float sel_raw = 0.0f;
  sel_e = 0;
  if (total > kMaxCand) {  // heavy ties at the threshold: k rounds over every code
    for (int j = 0; j < k; ++j) {
      uint32_t best = 0u;
      int bi = 0;
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if (code[i] > best) {  // strict: the lowest index wins ties
          best = code[i];
          bi = i;
        }
      const uint32_t top = __reduce_max_sync(kFull, best);
      const uint32_t win =
          __reduce_min_sync(kFull, (best == top) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu);
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if ((uint32_t)(lane + 32 * i) == win) code[i] = 0u;
      if (lane == j) {
        sel_e = (int)win;
        sel_raw = srow[win];
      }
    }
  } else {
    int pre = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, pre, o);
      if (lane >= o) pre += y;
    }
    pre -= c;
    // only the few candidate keys are visited; their codes are formed again
    // from the staged row (a candidate's rank is kept, so no mask applies)
    uint64_t* ckey = reinterpret_cast<uint64_t*>(cand);
    for (uint32_t m = cmask; m != 0u; m &= m - 1u) {
      const int e = lane + 32 * (__ffs(m) - 1);
      const uint32_t ce = order_code(__fadd_rn(srow[e], sbias[e]));
      ckey[pre] = ((uint64_t)ce << 32) | (uint64_t)(~(uint32_t)e);
      ++pre;
    }
    __syncwarp();
    uint32_t unused = 0u;
    select_ranked<false>(ckey, cand + 2 * kMaxCand, total, k, lane, sel_e, unused);
    if (lane < k) sel_raw = srow[sel_e];
  }

  if (renorm) {
    const float m = warp_max_f(lane < k ? sel_raw : -INFINITY);
    const double ex = (lane < k) ? exp((double)sel_raw - (double)m) : 0.0;
    const double den = warp_sum_d(ex);
    gate = (float)(ex * __drcp_rn(den));
  } else {
    float lm = -INFINITY;
#pragma unroll
    for (int i = 0; i < NK; ++i)
      if (lane + 32 * i < E) lm = fmaxf(lm, srow[lane + 32 * i]);
    const float m = warp_max_f(lm);
    double part = 0.0;
#pragma unroll
    for (int i = 0; i < NK; ++i)
      if (lane + 32 * i < E) part += exp((double)srow[lane + 32 * i] - (double)m);
    const double den = warp_sum_d(part);
    gate = (float)(exp((double)sel_raw - (double)m) * __drcp_rn(den));
  }
  return nan_tok;
}

// ---------------------------------------------------------------------------
// The fast form for staged rows without a rank limit: the same top-k, decided
// on the float keys themselves.  Lane l holds experts l, l+32, l+64, ... (so
// experts with neighbouring ids, which a skewed router often makes the
// popular ones, sit on different lanes and tau stays tight).  Float order is
// the key order here: +0 and -0 compare equal, as their folded codes do, and
// NaN is excluded up front.
//   1. lane maximum by three-input max.NaN: a NaN key makes it NaN, and one
//      NaN-propagating warp max per token then detects any NaN key;
//   2. tau = the k-th largest lane maximum (k rounds of an integer warp max on
//      order codes, lowered at most to the bottom of a 32-code bucket);
//   3. the keys >= tau (k to k+4 typically, at most 32 taken here) are
//      compacted by ballot rounds into shared memory as (value, expert);
//   4. candidate i's slot is the number of candidates with a strictly larger
//      value, read four at a time; with no two equal values that is the
//      exact order, and two equal values among the first k slots land on the
//      same slot, which the writer check below detects.
// A NaN key, more than 32 candidates or equal values at a slot below k take
// the exact code-based form (route_token_smem), so every result is the same
// bits as that form's.
constexpr int kFastMaxCand = 32;

__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float max2_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
__device__ __forceinline__ float warp_max_nan(float v) {
  float r;
  asm volatile("redux.sync.max.NaN.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Per-lane constant: bit i is set when key i (expert lane + 32 i) is < E.
template <int NK>
struct FastLanes {
  uint32_t vmask = 0u;
  __device__ void init(int E, int lane) {
    vmask = 0u;
#pragma unroll
    for (int i = 0; i < NK; ++i)
      if (lane + 32 * i < E) vmask |= 1u << i;
  }
};

// Selection only: true with lane j < k holding slot j's expert and raw logit,
// false when the token needs the exact form (nothing is decided then).
template <int NK>
__device__ __forceinline__ bool select_fast(const float* srow, const float* sbias, bool has_bias,
                                            int k, int lane, uint32_t* cand,
                                            const FastLanes<NK>& F, int& sel_e,
                                            float& sel_raw) {
  static_assert(NK >= 8 && NK <= 32, "the staged form");
  float key[NK];
  if (has_bias) {
#pragma unroll
    for (int i = 0; i < NK; ++i) {
      const int e = lane + 32 * i;
      key[i] = ((F.vmask >> i) & 1u) ? __fadd_rn(srow[e], sbias[e]) : -INFINITY;
    }
  } else if (F.vmask == (NK == 32 ? 0xffffffffu : (1u << NK) - 1u)) {
#pragma unroll
    for (int i = 0; i < NK; ++i) key[i] = srow[lane + 32 * i];
  } else {
#pragma unroll
    for (int i = 0; i < NK; ++i) key[i] = ((F.vmask >> i) & 1u) ? srow[lane + 32 * i] : -INFINITY;
  }
  // 1. lane maximum; any NaN key makes the warp maximum NaN
  float mm = key[0];
#pragma unroll
  for (int i = 1; i + 1 < NK; i += 2) mm = max3_nan(mm, key[i], key[i + 1]);
  mm = max2_nan(mm, key[NK - 1]);  // NK is even: the last key is left over
  const float wmax = warp_max_nan(mm);
  if (wmax != wmax) return false;
  // 2. tau: the k-th largest lane maximum, taken on order codes whose low 5
  //    bits are replaced by the lane (each code unique, so a round is one
  //    integer warp max and the holder clears its own); the truncation can
  //    only lower tau, to the smallest float of the truncated code, which
  //    still has k keys at or above it
  uint32_t m = (order_code(mm) & ~31u) | (uint32_t)(31 - lane);
  uint32_t top = 0u;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    top = __reduce_max_sync(kFull, m);
    m = (m == top) ? 0u : m;
  }
  // (codes below 2^23 are -inf, whose truncated code would read as a NaN)
  const float tau = top < 0x00800000u ? -INFINITY : code_float(top & ~31u);
  uint32_t cm = 0u;
#pragma unroll
  for (int i = 0; i < NK; ++i) cm |= (key[i] >= tau) ? (1u << i) : 0u;
  cm &= F.vmask;
  const int total = (int)__reduce_add_sync(kFull, (unsigned)__popc(cm));
  if (total > kFastMaxCand) return false;
  // 3. compaction by ballot rounds: (value, expert) of candidate p at cv[p], ce[p]
  float* cv = reinterpret_cast<float*>(cand);     // kFastMaxCand + 4 words
  int* ce = reinterpret_cast<int*>(cand + 64);     // kFastMaxCand words
  int* slot = reinterpret_cast<int*>(cand + 128);  // k words
  int base = 0;
#pragma unroll 1
  while (true) {
    const unsigned any = __ballot_sync(kFull, cm != 0u);
    if (any == 0u) break;
    if (cm != 0u) {
      const int e = lane + 32 * (__ffs(cm) - 1);
      const int p = base + __popc(any & lanemask_lt());
      cv[p] = has_bias ? __fadd_rn(srow[e], sbias[e]) : srow[e];
      ce[p] = e;
      cm &= cm - 1u;
    }
    base += __popc(any);
  }
  if (lane < 4) cv[total + lane] = -INFINITY;  // pads the last group of four
  __syncwarp();
  // 4. slots: candidates with a strictly larger value
  int n = 0;
  const float v = lane < total ? cv[lane] : INFINITY;
#pragma unroll 1
  for (int m0 = 0; m0 < total; m0 += 4) {
    const float4 q = *reinterpret_cast<const float4*>(cv + m0);
    n += (q.x > v) + (q.y > v) + (q.z > v) + (q.w > v);
  }
  const bool mine = lane < total && n < k;
  if (mine) slot[n] = lane;
  __syncwarp();
  const bool clash = mine && slot[n] != lane;
  if (__any_sync(kFull, clash)) {  // equal values among the first k
    __syncwarp();
    return false;
  }
  if (lane < k) {
    sel_e = ce[slot[lane]];
    sel_raw = srow[sel_e];
  }
  __syncwarp();  // the next token may overwrite the candidates
  return true;
}

// The exact code-based form, out of line: it runs for rare tokens only, and
// kept apart it does not raise the fast form's register count.
template <int NK>
__device__ __noinline__ int route_token_exact(const float* srow, const float* sbias, int t, int E,
                                              int k, int renorm, int lane, uint32_t* cand,
                                              int& sel_e, float& gate) {
  return route_token_smem<NK, false>(srow, sbias, t, E, k, renorm, lane, cand, sel_e, gate,
                                     RankLimit());
}

// Renormalised gates of one token whose slot j (j < k) sits on lane j: the
// softmax of the selected raw logits, as in the forms above.
__device__ __forceinline__ float gate_renorm(float sel_raw, int k, int lane) {
  const float m = warp_max_f(lane < k ? sel_raw : -INFINITY);
  const double ex = (lane < k) ? exp((double)sel_raw - (double)m) : 0.0;
  const double den = warp_sum_d(ex);
  return (float)(ex * __drcp_rn(den));
}

// The same for two tokens at once (k <= 16): token A's slots on lanes 0..15,
// token B's moved to lanes 16..31, each half reduced on its own, so one pass
// of the fp64 exponential and reciprocal serves both.  For k <= 16 the
// one-token form's first reduction step (across the halves) only adds zeros
// and -inf, so both give the same bits.  On return lane j < k holds A's slot
// j gate in ga and B's in gb.
__device__ __forceinline__ void gate_renorm_pair(float ra, float rb, int k, int lane, float& ga,
                                                 float& gb) {
  const float rb_hi = __shfl_sync(kFull, rb, lane & 15);
  const float x = lane < 16 ? ra : rb_hi;
  const bool act = (lane & 15) < k;
  float m = act ? x : -INFINITY;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  const double ex = act ? exp((double)x - (double)m) : 0.0;
  double den = ex;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) den += __shfl_xor_sync(kFull, den, o);
  const float g = (float)(ex * __drcp_rn(den));
  ga = g;
  gb = __shfl_sync(kFull, g, (lane + 16) & 31);
}

// Gates of one token from the staged row (renorm: the selected logits only;
// else the softmax over all E logits read at the selected experts).
__device__ __forceinline__ float gate_staged(const float* srow, float sel_raw, int E, int k,
                                             int renorm, int lane) {
  if (renorm) return gate_renorm(sel_raw, k, lane);
  float lm = -INFINITY;
  for (int e = lane; e < E; e += 32) lm = fmaxf(lm, srow[e]);
  const float m = warp_max_f(lm);
  double part = 0.0;
  for (int e = lane; e < E; e += 32) part += exp((double)srow[e] - (double)m);
  const double den = warp_sum_d(part);
  return (float)(exp((double)sel_raw - (double)m) * __drcp_rn(den));
}

}  // namespace moe
