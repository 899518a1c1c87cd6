/*
 * moe_oracle.c -- plain, slow, single-threaded CPU restatement of the MoE
 * token route / layout / dispatch / combine path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant
 * generator with the CUDA library: every rule below is written out again
 * from the pages' prose.
 *
 * Sources (page title, section):
 *   [A2A]  "19. All-to-all" (ai-from-scratch), opening section: each token
 *          carries a list of expert ids; dispatch ships the token's vector to
 *          the owners of those experts, combine ships the results back and
 *          mixes them.
 *   [BIAS] "19. All-to-all", section "Why the router can ruin your day":
 *          a per-expert bias, bumped by recent load, takes part in the top-k
 *          decision only, never in the mix weights; over-capacity tokens are
 *          dropped and treated as if they skipped that expert.
 *   [TWO]  "GPU MoE all-to-all" (aicassindra), section "Two collectives per
 *          layer, and what each one moves": k copies go out, k partial
 *          results come back, combine is the inverse permutation scaled by
 *          the router's gate weights; per-destination counts precede the
 *          payload.
 *   [BUCK] "GPU MoE all-to-all", section "Bucketing: cut the message count,
 *          not the byte count": sort rows by destination, build the offset
 *          table, each destination contiguous, counts kept on the device.
 *   [RAG]  "MoE All-to-All Dispatch and Ragged Routing", sections "Fixed
 *          Capacity vs. Ragged Routing" (capacity factor, rigid per-expert
 *          slots, overflow dropped; dropless ragged alternative) and
 *          "Returning Tokens to the Original GPU" (residual x + dx).
 *   [LAT]  "GPU MoE all-to-all", section "Latency-bound at decode,
 *          bandwidth-bound at prefill": lower-precision dispatch, since the
 *          activations feed a matmul that would cast them anyway.
 *   [OWN]  "Mixture-of-experts acceleration through overlap" (thecoregrid):
 *          remote-owner-aligned layout, every tile bound to one destination.
 *   [MSG]  "GPU MoE all-to-all", section "The message-size distribution is
 *          the whole story": an all-to-all over a group of ranks is one
 *          logical message per (sender, receiver) pair, whatever the batch.
 *   [FIRST] "Mixture-of-experts acceleration through overlap" (thecoregrid):
 *          remote-owner-aligned layout (each tile bound to one destination
 *          rank, sent as one contiguous write) and remote-first scheduling
 *          (the data bound for other GPUs is produced first).
 *   [DIAG] "GPU MoE all-to-all", section "How to tell whether the
 *          all-to-all is your bottleneck": replace the learned router by a
 *          uniform round-robin assignment to separate skew from the wire.
 *   [NODE] "19. All-to-all", opening section: each token is limited to at
 *          most 4 nodes so the slow hop stays bounded; section "Why Qwen3.8's
 *          512 experts is a systems statement": node-limited routing as an
 *          architectural constraint; "GPU MoE all-to-all", section "The node
 *          boundary is the design decision": a token whose top-k experts sit
 *          inside one node never crosses the NIC.  The pages give no group
 *          score; the one used here is the largest key on the rank.
 *   [OCP]  OCP 8-bit Floating Point Specification (OFP8), E4M3 format:
 *          exponent bias 7, 3 mantissa bits, no infinities, S.1111.111 is
 *          NaN, largest finite magnitude 448, smallest subnormal 2^-9.
 *
 * Precision: the pages fix none.  Decisions that turn floats into integers
 * (the top-k selection key, the e4m3 codes) are taken in fp32, the precision
 * the kernels decide in.  Everything else (gate softmax, combine sum) is
 * evaluated in fp64 and rounded once at the end.  The combine is also given
 * in the accumulation the hot path is specified with (binary32, fixed slot
 * order; orc_combine_f32), pinned against the fp64 sum by the binary32 error
 * bound and by hand-worked cases where the order decides the result.
 *
 * Parity pins: every function here is pinned by CPU tests (brute force,
 * closed forms, library special cases, hand-worked fixtures); none is
 * "parity unpinned".
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared (see oracle/build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_BAD_ARG 1
#define ORC_BAD_ID 2

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
double orc_bf16_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static float bf16_to_float(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Round a real number (held exactly in a double) to the nearest bf16, ties to
 * even, in ONE rounding.  bf16 keeps 8 significant bits, exponent range of
 * binary32, subnormal quantum 2^-133.  Overflow past the largest finite value
 * (plus half a quantum) gives infinity, as round-to-nearest does. */
uint16_t orc_double_to_bf16(double v) {
  if (isnan(v)) return 0x7FC0;
  uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
  double a = fabs(v);
  if (a == 0.0) return sign;
  int e2;
  (void)frexp(a, &e2);          /* a = m * 2^e2, m in [0.5, 1) */
  int lead = e2 - 1;            /* a in [2^lead, 2^(lead+1)) */
  int qexp = lead - 7;          /* quantum of an 8-significant-bit number */
  if (qexp < -133) qexp = -133; /* subnormal range */
  double r = nearbyint(ldexp(a, -qexp)); /* default mode: nearest, ties even */
  double q = ldexp(r, qexp);
  const double maxfin = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
  if (q > maxfin) return (uint16_t)(sign | 0x7F80);
  float f = (float)q;           /* exact: q has <= 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFF));
}

/* Round a binary32 to bf16, nearest-even.  A float is exactly a double, so
 * this is the same single rounding. */
static uint16_t float_to_bf16(float f) { return orc_double_to_bf16((double)f); }

/* [OCP] E4M3 value of a code. */
double orc_e4m3_decode(uint8_t c) {
  int s = (c >> 7) & 1;
  int E = (c >> 3) & 0xF;
  int M = c & 0x7;
  if (E == 15 && M == 7) return NAN;
  double mag;
  if (E == 0) mag = ldexp((double)M / 8.0, -6);          /* subnormal */
  else mag = ldexp(1.0 + (double)M / 8.0, E - 7);        /* normal */
  return s ? -mag : mag;
}

/* [OCP] Encode a binary32 to E4M3: round to nearest, ties to even; finite
 * values beyond 448 (and infinities) saturate to +-448; NaN stays NaN. */
uint8_t orc_e4m3_encode_satfinite(float f) {
  if (isnan(f)) return 0x7F;
  uint8_t s = signbit(f) ? 0x80 : 0x00;
  double a = fabs((double)f);
  if (a >= 448.0) return (uint8_t)(s | 0x7E);
  if (a == 0.0) return s;
  int e2;
  (void)frexp(a, &e2);
  int lead = e2 - 1;
  int qexp = lead - 3;            /* 4 significant bits for normals */
  if (qexp < -9) qexp = -9;       /* subnormal quantum 2^-9 */
  double r = nearbyint(ldexp(a, -qexp));
  double q = ldexp(r, qexp);      /* the rounded magnitude, <= 448 here */
  if (q > 448.0) q = 448.0;       /* cannot happen below 448, kept for clarity */
  if (q == 0.0) return s;
  (void)frexp(q, &e2);
  lead = e2 - 1;
  if (lead < -6) {                /* subnormal: E = 0, value = M * 2^-9 */
    int M = (int)ldexp(q, 9);
    return (uint8_t)(s | M);
  }
  int E = lead + 7;
  int M = (int)(ldexp(q, -lead) * 8.0 - 8.0);
  return (uint8_t)(s | (E << 3) | M);
}

/* ------------------------------------------------------------------------ */
/* Step 1: route.  [A2A], [BIAS]                                             */
/* ------------------------------------------------------------------------ */

/* For each token t:
 *   key_e  = logit[t,e] + bias[e], one binary32 addition (bias NULL: 0);
 *   slots  = the k experts with the largest keys, slot j the j-th largest;
 *            equal keys: the lower expert id first (+0 and -0 are equal);
 *   gates  = softmax of the RAW logits (the bias never enters the weights),
 *            over the k selected experts when renorm != 0, else over all E
 *            experts and read at the selected ones.  Evaluated in fp64 and
 *            rounded to binary32 once.
 * Returns ORC_BAD_ARG on bad sizes. */
int orc_route(int T, int E, int k, int renorm, const float* logits, const float* bias,
              int32_t* ids, float* gates) {
  if (T < 0 || E < 1 || k < 1 || k > E) return ORC_BAD_ARG;
  float* key = (float*)malloc(sizeof(float) * (size_t)E);
  unsigned char* taken = (unsigned char*)malloc((size_t)E);
  if (!key || !taken) { free(key); free(taken); return ORC_BAD_ARG; }
  for (int t = 0; t < T; ++t) {
    const float* lg = logits + (size_t)t * E;
    for (int e = 0; e < E; ++e) {
      float b = bias ? bias[e] : 0.0f;
      key[e] = lg[e] + b;
      taken[e] = 0;
    }
    /* k rounds of "largest remaining key, lowest id among equals" */
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || key[e] > key[best]) best = e; /* strict: keeps lower id on ties */
      }
      taken[best] = 1;
      ids[(size_t)t * k + j] = best;
    }
    /* gates from the raw logits */
    double m = -INFINITY;
    if (renorm) {
      for (int j = 0; j < k; ++j) {
        double l = (double)lg[ids[(size_t)t * k + j]];
        if (l > m) m = l;
      }
      double den = 0.0;
      for (int j = 0; j < k; ++j) den += exp((double)lg[ids[(size_t)t * k + j]] - m);
      for (int j = 0; j < k; ++j)
        gates[(size_t)t * k + j] = (float)(exp((double)lg[ids[(size_t)t * k + j]] - m) / den);
    } else {
      for (int e = 0; e < E; ++e)
        if ((double)lg[e] > m) m = (double)lg[e];
      double den = 0.0;
      for (int e = 0; e < E; ++e) den += exp((double)lg[e] - m);
      for (int j = 0; j < k; ++j)
        gates[(size_t)t * k + j] = (float)(exp((double)lg[ids[(size_t)t * k + j]] - m) / den);
    }
  }
  free(key);
  free(taken);
  return ORC_OK;
}

/* Rank-limited route.  [NODE], [BIAS]
 * As orc_route, except that each token's experts come from at most M of the
 * R ranks (expert e lives on rank e / (E/R)):
 *   score_r = max over the experts e of rank r of key_e;
 *   the M ranks with the largest scores are eligible (equal scores: the
 *   lower rank id first);
 *   slots  = the k largest keys among the eligible ranks' experts (equal
 *            keys: the lower expert id first);
 *   gates  = as orc_route (raw logits; renorm over the k selected, else the
 *            softmax over all E read at the selected ones).
 * Needs 1 <= M, and k <= M * (E/R) so that k experts are eligible.  M >= R
 * is the unrestricted route. */
int orc_route_limited(int T, int E, int k, int R, int M, int renorm, const float* logits,
                      const float* bias, int32_t* ids, float* gates) {
  if (T < 0 || E < 1 || k < 1 || k > E || R < 1 || E % R != 0 || M < 1) return ORC_BAD_ARG;
  const int Er = E / R;
  if (M < R && k > M * Er) return ORC_BAD_ARG;
  float* key = (float*)malloc(sizeof(float) * (size_t)E);
  unsigned char* taken = (unsigned char*)malloc((size_t)E);
  float* score = (float*)malloc(sizeof(float) * (size_t)R);
  unsigned char* chosen = (unsigned char*)malloc((size_t)R);
  if (!key || !taken || !score || !chosen) {
    free(key); free(taken); free(score); free(chosen);
    return ORC_BAD_ARG;
  }
  for (int t = 0; t < T; ++t) {
    const float* lg = logits + (size_t)t * E;
    for (int e = 0; e < E; ++e) {
      key[e] = lg[e] + (bias ? bias[e] : 0.0f);
      taken[e] = 0;
    }
    if (M < R) {
      /* group score per rank, then the M best ranks */
      for (int r = 0; r < R; ++r) {
        score[r] = key[r * Er];
        for (int e = r * Er + 1; e < (r + 1) * Er; ++e)
          if (key[e] > score[r]) score[r] = key[e];
        chosen[r] = 0;
      }
      for (int m = 0; m < M; ++m) {
        int best = -1;
        for (int r = 0; r < R; ++r) {
          if (chosen[r]) continue;
          if (best < 0 || score[r] > score[best]) best = r; /* strict: lower id on ties */
        }
        chosen[best] = 1;
      }
      /* experts of the other ranks cannot be selected */
      for (int e = 0; e < E; ++e)
        if (!chosen[e / Er]) taken[e] = 1;
    }
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || key[e] > key[best]) best = e;
      }
      taken[best] = 1;
      ids[(size_t)t * k + j] = best;
    }
    double m = -INFINITY;
    if (renorm) {
      for (int j = 0; j < k; ++j) {
        double l = (double)lg[ids[(size_t)t * k + j]];
        if (l > m) m = l;
      }
      double den = 0.0;
      for (int j = 0; j < k; ++j) den += exp((double)lg[ids[(size_t)t * k + j]] - m);
      for (int j = 0; j < k; ++j)
        gates[(size_t)t * k + j] = (float)(exp((double)lg[ids[(size_t)t * k + j]] - m) / den);
    } else {
      for (int e = 0; e < E; ++e)
        if ((double)lg[e] > m) m = (double)lg[e];
      double den = 0.0;
      for (int e = 0; e < E; ++e) den += exp((double)lg[e] - m);
      for (int j = 0; j < k; ++j)
        gates[(size_t)t * k + j] = (float)(exp((double)lg[ids[(size_t)t * k + j]] - m) / den);
    }
  }
  free(key); free(taken); free(score); free(chosen);
  return ORC_OK;
}

/* Aux-loss-free balancing: the per-expert bias update.  [BIAS]
 * After a batch with load_e = counts[e] assignments per expert (before any
 * drop) and mean = T*k/E, every bias moves by gamma towards balance:
 *   b_e <- b_e + gamma * sign(mean - load_e)
 * (an under-loaded expert's bias rises, an over-loaded one's falls, an
 * expert exactly at the mean keeps its bias).  The sign is taken exactly, in
 * integers: sign(T*k - E*load_e).  The update is one binary32 addition of
 * +gamma, -gamma or nothing.  The pages give neither gamma nor the sign
 * rule's form beyond "bump up or down based on recent load". */
void orc_bias_update(int E, int64_t assignments, const int32_t* counts, float gamma,
                     const float* bias_in, float* bias_out) {
  for (int e = 0; e < E; ++e) {
    const int64_t d = assignments - (int64_t)E * counts[e];
    if (d > 0)
      bias_out[e] = bias_in[e] + gamma;
    else if (d < 0)
      bias_out[e] = bias_in[e] - gamma;
    else
      bias_out[e] = bias_in[e];
  }
}

/* ------------------------------------------------------------------------ */
/* Steps 2-3: count histogram and layout.  [TWO], [BUCK], [RAG], [OWN]       */
/* ------------------------------------------------------------------------ */

/* Rows the layout holds: dropless T*k + E*(align-1) (worst-case padding, a
 * static bound so nothing waits on the counts), capacity E*C. */
int64_t orc_layout_rows(int T, int E, int k, int capacity, int align) {
  if (capacity > 0) return (int64_t)E * capacity;
  return (int64_t)T * k + (int64_t)E * (align - 1);
}

/* Expert e lives on logical rank e / (E/R); ranks own consecutive experts, so
 * a rank's rows form one contiguous slice of the layout.
 *
 *   counts[e]      number of (t,j) with ids[t,j] == e (before any drop)
 *   expert_off[e]  first row of expert e's segment; expert_off[E] = rows used
 *                  dropless: segments of round_up(counts[e], align) rows
 *                  capacity: segments of exactly C rows (expert_off[e] = e*C)
 *   rank_off[r]    = expert_off[r*E/R]; rank_off[R] = expert_off[E]
 *   rank_counts[r] rows of rank r's slice that hold a token (padding and
 *                  dropped assignments excluded)
 *   dst_pos[t,j]   row of assignment (t,j), -1 if dropped
 *   src_idx[p]     t*k + j of the assignment in row p, -1 if the row is empty
 *
 * Within an expert, rows follow token order (t ascending); in capacity mode
 * the first C assignments in that order are kept and the rest dropped. */
int orc_layout(int T, int E, int k, int R, int capacity, int align, const int32_t* ids,
               int32_t* counts, int32_t* expert_off, int32_t* rank_off, int32_t* rank_counts,
               int32_t* dst_pos, int32_t* src_idx) {
  if (T < 0 || E < 1 || k < 1 || k > E || R < 1 || E % R != 0 || capacity < 0 || align < 1)
    return ORC_BAD_ARG;
  for (size_t i = 0; i < (size_t)T * k; ++i)
    if (ids[i] < 0 || ids[i] >= E) return ORC_BAD_ID;
  int64_t N = orc_layout_rows(T, E, k, capacity, align);
  int Er = E / R;

  /* histogram */
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (size_t i = 0; i < (size_t)T * k; ++i) counts[ids[i]] += 1;

  /* exclusive scan over experts -> segment starts */
  expert_off[0] = 0;
  for (int e = 0; e < E; ++e) {
    int32_t seg;
    if (capacity > 0) seg = capacity;
    else seg = ((counts[e] + align - 1) / align) * align;
    expert_off[e + 1] = expert_off[e] + seg;
  }
  for (int r = 0; r < R; ++r) {
    rank_off[r] = expert_off[r * Er];
    int32_t kept = 0;
    for (int e = r * Er; e < (r + 1) * Er; ++e)
      kept += (capacity > 0 && counts[e] > capacity) ? capacity : counts[e];
    rank_counts[r] = kept;
  }
  rank_off[R] = expert_off[E];

  /* positions: walk assignments in token order with a cursor per expert */
  for (int64_t p = 0; p < N; ++p) src_idx[p] = -1;
  int32_t* cursor = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  if (!cursor) return ORC_BAD_ARG;
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      size_t i = (size_t)t * k + j;
      int e = ids[i];
      int32_t c = cursor[e]++;
      if (capacity > 0 && c >= capacity) {
        dst_pos[i] = -1; /* dropped: as if the token skipped this expert */
        continue;
      }
      int32_t p = expert_off[e] + c;
      dst_pos[i] = p;
      src_idx[p] = (int32_t)i;
    }
  }
  free(cursor);
  return ORC_OK;
}

/* Per-source-rank layout: the metadata and receive buffers a ragged
 * all-to-all posts.  [TWO], [MSG], [RAG], [OWN]
 *
 * The T tokens are split into R source shards of Ts = ceil(T/R) consecutive
 * tokens (shard s holds tokens s*Ts .. s*Ts+Ts-1; trailing shards may be short
 * or empty).  Expert e lives on rank r = e / (E/R) as before.  The rows are
 * the receive side of the exchange: ordered by destination rank r, then
 * source shard s, then expert e (all ascending), then token order; segment
 * (r, s, e) holds the assignments from shard s to expert e.
 *
 *   src_counts[s*E + e]   assignments of shard s to expert e (before drops)
 *   seg_off[i]            first row of segment i = (r*R + s)*(E/R) + (e - r*(E/R));
 *                         dropless: round_up(src_counts, align) rows per segment;
 *                         capacity: exactly C rows per segment (per-sender-
 *                         expert slots); seg_off[R*E] = rows used
 *   pair_counts[s*R + r]  rows kept from shard s for rank r (the message size)
 *   rank_off[r]           = seg_off[r*R*(E/R)] (rank r's slice); rank_off[R] = seg_off[R*E]
 *   rank_counts[r]        rows kept for rank r from all shards
 *   dst_pos, src_idx      as in orc_layout; capacity keeps the first C
 *                         assignments of each (shard, expert) in token order
 */
int64_t orc_layout_src_rows(int T, int E, int k, int R, int capacity, int align) {
  if (capacity > 0) return (int64_t)R * E * capacity;
  return (int64_t)T * k + (int64_t)R * E * (align - 1);
}

int orc_layout_src(int T, int E, int k, int R, int capacity, int align, const int32_t* ids,
                   int32_t* src_counts, int32_t* seg_off, int32_t* pair_counts,
                   int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                   int32_t* src_idx) {
  if (T < 0 || E < 1 || k < 1 || k > E || R < 1 || E % R != 0 || capacity < 0 || align < 1)
    return ORC_BAD_ARG;
  for (size_t i = 0; i < (size_t)T * k; ++i)
    if (ids[i] < 0 || ids[i] >= E) return ORC_BAD_ID;
  const int64_t N = orc_layout_src_rows(T, E, k, R, capacity, align);
  const int Er = E / R;
  const int Ts = T > 0 ? (T + R - 1) / R : 1;

  /* counts per (source shard, expert) */
  for (int s = 0; s < R; ++s)
    for (int e = 0; e < E; ++e) src_counts[s * E + e] = 0;
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) src_counts[(t / Ts) * E + ids[(size_t)t * k + j]] += 1;

  /* segments in (rank, shard, expert) order; exclusive scan of their sizes */
  int32_t run = 0;
  for (int r = 0; r < R; ++r)
    for (int s = 0; s < R; ++s)
      for (int el = 0; el < Er; ++el) {
        const int e = r * Er + el;
        const int32_t c = src_counts[s * E + e];
        seg_off[(r * R + s) * Er + el] = run;
        run += capacity > 0 ? capacity : ((c + align - 1) / align) * align;
      }
  seg_off[R * E] = run;

  /* message sizes and rank slices */
  for (int s = 0; s < R; ++s)
    for (int r = 0; r < R; ++r) {
      int32_t kept = 0;
      for (int e = r * Er; e < (r + 1) * Er; ++e) {
        const int32_t c = src_counts[s * E + e];
        kept += (capacity > 0 && c > capacity) ? capacity : c;
      }
      pair_counts[s * R + r] = kept;
    }
  for (int r = 0; r < R; ++r) {
    rank_off[r] = seg_off[r * R * Er];
    int32_t kept = 0;
    for (int s = 0; s < R; ++s) kept += pair_counts[s * R + r];
    rank_counts[r] = kept;
  }
  rank_off[R] = seg_off[R * E];

  /* positions: token order, one cursor per (shard, expert) */
  for (int64_t p = 0; p < N; ++p) src_idx[p] = -1;
  int32_t* cursor = (int32_t*)calloc((size_t)R * E, sizeof(int32_t));
  if (!cursor) return ORC_BAD_ARG;
  for (int t = 0; t < T; ++t) {
    const int s = t / Ts;
    for (int j = 0; j < k; ++j) {
      const size_t i = (size_t)t * k + j;
      const int e = ids[i];
      const int r = e / Er;
      const int32_t c = cursor[s * E + e]++;
      if (capacity > 0 && c >= capacity) {
        dst_pos[i] = -1;
        continue;
      }
      const int32_t p = seg_off[(r * R + s) * Er + (e - r * Er)] + c;
      dst_pos[i] = p;
      src_idx[p] = (int32_t)i;
    }
  }
  free(cursor);
  return ORC_OK;
}

/* Remote-first, tile-aligned layout.  [FIRST], [OWN], [RAG]
 * As orc_layout, except for the order of the rank slices: seen from rank
 * `home` (the GPU the batch lives on), the slices of the other ranks come
 * first, in the order home+1, home+2, ... (mod R), and home's own slice
 * last.  Experts keep their order inside a slice and assignments their
 * token order inside an expert.  expert_off[e] is the first row of expert e
 * (no longer increasing in e); expert_off[E] = rows used; rank_off[r] =
 * expert_off[r*E/R], rank_off[R] = rows used.  With align = A every expert
 * segment is a whole number of A-row tiles, each inside one expert and so
 * bound to one destination rank:
 *   tile_expert[i]  expert owning rows i*A .. i*A+A-1, -1 past the rows
 *                   used; N/A entries (N = orc_layout_rows).
 * In capacity mode the tiles are C rows' worth: A = align = 1 and every row
 * is a tile. */
int orc_layout_remote_first(int T, int E, int k, int R, int capacity, int align, int home,
                            const int32_t* ids, int32_t* counts, int32_t* expert_off,
                            int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                            int32_t* src_idx, int32_t* tile_expert) {
  if (T < 0 || E < 1 || k < 1 || k > E || R < 1 || E % R != 0 || capacity < 0 || align < 1 ||
      home < 0 || home >= R)
    return ORC_BAD_ARG;
  for (size_t i = 0; i < (size_t)T * k; ++i)
    if (ids[i] < 0 || ids[i] >= E) return ORC_BAD_ID;
  const int64_t N = orc_layout_rows(T, E, k, capacity, align);
  const int Er = E / R;

  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (size_t i = 0; i < (size_t)T * k; ++i) counts[ids[i]] += 1;

  /* segments in slice order: ranks home+1, ..., home+R (mod R), experts ascending */
  int32_t run = 0;
  for (int q = 1; q <= R; ++q) {
    const int r = (home + q) % R;
    for (int e = r * Er; e < (r + 1) * Er; ++e) {
      expert_off[e] = run;
      run += capacity > 0 ? capacity : ((counts[e] + align - 1) / align) * align;
    }
  }
  expert_off[E] = run;
  for (int r = 0; r < R; ++r) {
    rank_off[r] = expert_off[r * Er];
    int32_t kept = 0;
    for (int e = r * Er; e < (r + 1) * Er; ++e)
      kept += (capacity > 0 && counts[e] > capacity) ? capacity : counts[e];
    rank_counts[r] = kept;
  }
  rank_off[R] = expert_off[E];

  for (int64_t p = 0; p < N; ++p) src_idx[p] = -1;
  int32_t* cursor = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  if (!cursor) return ORC_BAD_ARG;
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const size_t i = (size_t)t * k + j;
      const int e = ids[i];
      const int32_t c = cursor[e]++;
      if (capacity > 0 && c >= capacity) {
        dst_pos[i] = -1;
        continue;
      }
      dst_pos[i] = expert_off[e] + c;
      src_idx[expert_off[e] + c] = (int32_t)i;
    }
  free(cursor);

  /* tile -> expert: walk the segments in slice order */
  for (int64_t i = 0; i < N / align; ++i) tile_expert[i] = -1;
  for (int e = 0; e < E; ++e) {
    const int32_t seg = capacity > 0 ? capacity : ((counts[e] + align - 1) / align) * align;
    for (int32_t row = expert_off[e]; row < expert_off[e] + seg; row += align)
      tile_expert[row / align] = e;
  }
  return ORC_OK;
}

/* Round-robin router: the diagnostic that replaces the learned router.
 * [DIAG]  ids[t,j] = (t*k + j) mod E (k distinct experts per token since
 * k <= E; every expert gets T*k/E assignments when E divides T*k), gates all
 * 1/k (rounded to binary32 once). */
void orc_route_round_robin(int T, int E, int k, int32_t* ids, float* gates) {
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      ids[(size_t)t * k + j] = (int32_t)(((int64_t)t * k + j) % E);
      gates[(size_t)t * k + j] = (float)(1.0 / (double)k);
    }
}

/* ------------------------------------------------------------------------ */
/* Step 4: dispatch.  [TWO], [BUCK], [LAT]                                   */
/* ------------------------------------------------------------------------ */

/* bf16: row dst_pos[t,j] of out is a copy of row t of x. */
void orc_dispatch_bf16(int T, int H, int k, const uint16_t* x, const int32_t* dst_pos,
                       uint16_t* out) {
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int32_t p = dst_pos[(size_t)t * k + j];
      if (p < 0) continue;
      memcpy(out + (size_t)p * H, x + (size_t)t * H, sizeof(uint16_t) * (size_t)H);
    }
}

/* FP8 quantisation of one token row, per 128-channel block b:
 *   amax_b = max |x_c| (exact in binary32)
 *   amax_b == 0:  all codes 0, scale 0
 *   otherwise:    inv = 448 / amax_b and scale_b = amax_b / 448 (binary32,
 *                 correctly rounded), q_c = e4m3(x_c * inv) with one binary32
 *                 multiply, nearest-even, saturating at +-448.
 * Dequantised value: decode(q_c) * scale_b. */
void orc_quantize_row_fp8(int H, const uint16_t* xrow, uint8_t* qrow, float* srow) {
  for (int b = 0; b < H / 128; ++b) {
    float amax = 0.0f;
    for (int c = 0; c < 128; ++c) {
      float v = fabsf(bf16_to_float(xrow[b * 128 + c]));
      if (v > amax) amax = v;
    }
    if (amax == 0.0f) {
      for (int c = 0; c < 128; ++c) qrow[b * 128 + c] = 0;
      srow[b] = 0.0f;
      continue;
    }
    float inv = 448.0f / amax;
    float scale = amax / 448.0f;
    for (int c = 0; c < 128; ++c) {
      float v = bf16_to_float(xrow[b * 128 + c]) * inv;
      qrow[b * 128 + c] = orc_e4m3_encode_satfinite(v);
    }
    srow[b] = scale;
  }
}

/* FP8 dispatch: every kept copy of token t gets the same codes and scales. */
void orc_dispatch_fp8(int T, int H, int k, const uint16_t* x, const int32_t* dst_pos,
                      uint8_t* out, float* scales) {
  int nb = H / 128;
  uint8_t* q = (uint8_t*)malloc((size_t)H);
  float* s = (float*)malloc(sizeof(float) * (size_t)nb);
  for (int t = 0; t < T; ++t) {
    orc_quantize_row_fp8(H, x + (size_t)t * H, q, s);
    for (int j = 0; j < k; ++j) {
      int32_t p = dst_pos[(size_t)t * k + j];
      if (p < 0) continue;
      memcpy(out + (size_t)p * H, q, (size_t)H);
      memcpy(scales + (size_t)p * nb, s, sizeof(float) * (size_t)nb);
    }
  }
  free(q);
  free(s);
}

/* ------------------------------------------------------------------------ */
/* Step 5: combine.  [TWO], [RAG], [BIAS]                                    */
/* ------------------------------------------------------------------------ */

/* out[t,c] = bf16( sum_{j kept} gates[t,j] * y[dst_pos[t,j], c]
 *                  (+ shared[t,c]) (+ residual[t,c]) )
 * The sum is taken in fp64 (every product of a binary32 gate and a bf16 value
 * is exact there) and rounded to bf16 once.  A dropped slot (dst_pos -1)
 * contributes nothing and the other gates are left as they are.  tokens ==
 * NULL means all tokens; otherwise only the listed tokens' rows of out are
 * written. */
void orc_combine(int T, int H, int k, const uint16_t* y, const int32_t* dst_pos,
                 const float* gates, const uint16_t* shared, const uint16_t* residual,
                 uint16_t* out, const int32_t* tokens, int n_tokens) {
  int n = tokens ? n_tokens : T;
  for (int i = 0; i < n; ++i) {
    int t = tokens ? tokens[i] : i;
    for (int c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) {
        int32_t p = dst_pos[(size_t)t * k + j];
        if (p < 0) continue;
        acc += (double)gates[(size_t)t * k + j] * orc_bf16_to_double(y[(size_t)p * H + c]);
      }
      if (shared) acc += orc_bf16_to_double(shared[(size_t)t * H + c]);
      if (residual) acc += orc_bf16_to_double(residual[(size_t)t * H + c]);
      out[(size_t)t * H + c] = orc_double_to_bf16(acc);
    }
  }
}

/* The same sum accumulated in binary32 in a fixed order: acc = +0; for each
 * kept slot j = 0..k-1, acc = fmaf(gates[t,j], y[dst_pos[t,j], c], acc) (one
 * fused multiply-add, one rounding); then acc = acc + shared[t,c]; then acc =
 * acc + residual[t,c] (one binary32 addition each); out = bf16 of acc, nearest
 * even.  Each step rounds once to binary32 (unit roundoff 2^-24), so with n
 * steps |acc - exact sum| <= n * 2^-24 * (1+2^-24)^n * (sum of the terms'
 * magnitudes); that difference decides the bf16 rounding where the exact sum
 * lies at or next to a bf16 midpoint, and dominates where the terms cancel.
 * Arguments as orc_combine. */
void orc_combine_f32(int T, int H, int k, const uint16_t* y, const int32_t* dst_pos,
                     const float* gates, const uint16_t* shared, const uint16_t* residual,
                     uint16_t* out, const int32_t* tokens, int n_tokens) {
  int n = tokens ? n_tokens : T;
  for (int i = 0; i < n; ++i) {
    int t = tokens ? tokens[i] : i;
    for (int c = 0; c < H; ++c) {
      float acc = 0.0f;
      for (int j = 0; j < k; ++j) {
        int32_t p = dst_pos[(size_t)t * k + j];
        if (p < 0) continue;
        acc = fmaf(gates[(size_t)t * k + j], bf16_to_float(y[(size_t)p * H + c]), acc);
      }
      if (shared) acc = acc + bf16_to_float(shared[(size_t)t * H + c]);
      if (residual) acc = acc + bf16_to_float(residual[(size_t)t * H + c]);
      out[(size_t)t * H + c] = float_to_bf16(acc);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Expert stand-ins used by the tests between dispatch and combine.  They    */
/* are not part of the path (the expert FFN is out of scope).                */
/* ------------------------------------------------------------------------ */

/* Row p of expert e scaled by (e+1)/E: bf16( x * ((float)(e+1)/(float)E) ),
 * one binary32 multiply. Rows outside every expert's used range are left. */
void orc_expert_scale(int E, int H, const int32_t* expert_off, const int32_t* counts,
                      int capacity, const uint16_t* xd, uint16_t* y) {
  for (int e = 0; e < E; ++e) {
    float s = (float)(e + 1) / (float)E;
    int32_t used = counts[e];
    if (capacity > 0 && used > capacity) used = capacity;
    for (int32_t r = 0; r < used; ++r) {
      size_t p = (size_t)(expert_off[e] + r);
      for (int c = 0; c < H; ++c)
        y[p * H + c] = float_to_bf16(bf16_to_float(xd[p * H + c]) * s);
    }
  }
}

/* Dequantise FP8 rows: bf16( decode(q) * scale ), one binary32 multiply. */
void orc_dequant_fp8(int64_t rows, int H, const uint8_t* q, const float* scales, uint16_t* y) {
  int nb = H / 128;
  for (int64_t p = 0; p < rows; ++p)
    for (int c = 0; c < H; ++c) {
      float v = (float)orc_e4m3_decode(q[p * H + c]);
      y[p * H + c] = float_to_bf16(v * scales[p * nb + c / 128]);
    }
}
