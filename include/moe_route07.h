/*
 * moe_route07.h -- C ABI of the on-GPU MoE token route / layout / dispatch /
 * combine path (NVIDIA B200, sm_100a).
 *
 * The four steps are the data-parallel part of the expert-parallel exchange
 * that the following pages describe:
 *   "GPU MoE all-to-all" (aicassindra): section "Two collectives per layer,
 *      and what each one moves" (dispatch replicates each token to its k
 *      experts, combine is the inverse permutation scaled by the gate weights,
 *      per-destination counts travel before the payload) and section
 *      "Bucketing: cut the message count, not the byte count" (sort rows by
 *      destination, build the offset table, keep counts on the device);
 *   "19. All-to-all" (ai-from-scratch): section "Why the router can ruin your
 *      day" (a per-expert bias used only for the top-k decision; tokens over
 *      capacity are dropped as if they skipped the expert);
 *   "MoE All-to-All Dispatch and Ragged Routing": section "Fixed Capacity vs.
 *      Ragged Routing" (capacity factor with drops, or dropless ragged
 *      layout) and section "Returning Tokens to the Original GPU" (x + dx);
 *   "Mixture-of-experts acceleration through overlap" (thecoregrid): the
 *      remote-owner-aligned layout (every row band bound to one destination).
 *
 * Besides the four steps (moe_route, moe_layout, moe_dispatch, moe_combine,
 * and the fused moe_route_layout / moe_route_layout_dispatch): the
 * per-source-rank layout of a ragged exchange (moe_layout_src), rank-limited
 * routing (moe_route_limited), the aux-loss-free bias update
 * (moe_bias_update), the remote-first tile-aligned layout
 * (moe_layout_remote_first), the round-robin router diagnostic
 * (moe_route_round_robin), an allocation-free layout (moe_layout_noalloc) and
 * a self-test of the kernels' failure path (moe_selftest_wait_timeout).
 *
 * Everything runs on one GPU.  The R "ranks" are logical partitions of the
 * dispatched buffer: expert e belongs to rank e / (E/R), and each rank's rows
 * form one contiguous slice.
 *
 * Conventions for every call:
 *  - All pointers except `shape` are DEVICE pointers owned by the caller; the
 *    library allocates nothing and keeps no state between calls (beyond
 *    host-side caches of launch parameters, and the static array of
 *    moe_layout_noalloc).
 *  - Calls are asynchronous on `stream` (NULL = legacy default stream).  Only
 *    moe_get_device_error synchronises.
 *  - Arguments are checked on the host first; on MOE_ERR_INVALID_ARG nothing
 *    is launched and no buffer is touched.
 *  - Problems found by the kernels (an expert id or row outside its range, a
 *    NaN routing key, a wait that gave up) never trap: the kernel records the
 *    first one in the workspace's error word and skips the offending element.
 *    moe_get_device_error reads and clears it.
 *  - A launch failure returns MOE_ERR_CUDA.
 *  - One workspace serves one stream at a time; calls that share a workspace
 *    must be ordered on the device (same stream, or event-ordered).
 */
#ifndef MOE_ROUTE07_H
#define MOE_ROUTE07_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* host check failed; nothing launched */
  MOE_ERR_UNSUPPORTED = 2,    /* valid request outside what this library supports */
  MOE_ERR_WORKSPACE = 3,      /* workspace NULL, misaligned or too small */
  MOE_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_RANGE = 5,   /* device: expert id or row index out of range */
  MOE_ERR_DEVICE_TIMEOUT = 6, /* device: a bounded wait gave up */
  MOE_ERR_DEVICE_NAN = 7      /* device: a routing key was NaN */
} moe_status_t;

/* flags */
#define MOE_F_RENORM 0x1u /* gates: softmax over the k selected experts (else over all E) */
#define MOE_F_FP8 0x2u    /* dispatch writes e4m3 codes + per-128-channel fp32 scales */
#define MOE_F_SRC_LAYOUT 0x4u /* rows follow the per-source-rank layout (moe_layout_src) */

/* Problem description (host memory).
 *   tokens   T >= 0
 *   hidden   H, multiple of 8 (bf16 rows of 16-byte multiples); multiple of
 *            128 with MOE_F_FP8
 *   experts  E, 1..1024, multiple of ranks
 *   k        slots per token, 1..min(E, 32)
 *   ranks    R >= 1 logical EP ranks (E/R consecutive experts each)
 *   capacity 0: dropless; C > 0: every expert owns exactly C rows and keeps
 *            its first C assignments in token order
 *   align    >= 1: dropless segments are rounded up to a multiple of align
 *            rows (must be 1 in capacity mode)
 *   flags    MOE_F_* bits
 * Limits: T*k < 2^30, and the layout's row count below 2^31. */
typedef struct {
  int32_t tokens, hidden, experts, k, ranks;
  int32_t capacity;
  int32_t align;
  uint32_t flags;
} moe_shape_t;

/* Rows N of the dispatched buffer: dropless T*k + E*(align-1), capacity E*C;
 * with MOE_F_SRC_LAYOUT dropless T*k + R*E*(align-1), capacity R*E*C.  A
 * static bound, so buffers are sized without reading counts back.  Returns -1
 * for an invalid shape. */
int64_t moe_layout_rows(const moe_shape_t* shape);

/* Bytes of device workspace the calls need for `shape` (error word, the
 * layout's counters and its per-tile prefix table).  0 for an invalid shape.
 * A workspace sized for one shape serves any shape whose requirement is not
 * larger. */
size_t moe_workspace_bytes(const moe_shape_t* shape);

/* Zero-fill a workspace (cudaMemsetAsync on `stream`).  Required once before
 * the workspace's first use, and again after a call returned MOE_ERR_CUDA;
 * every successful call leaves it ready for the next one. */
moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Step 1 -- route ("19. All-to-all", section "Why the router can ruin your
 * day").  For each token t:
 *   key[e]   = logits[t,e] + bias[e]       (one fp32 add; bias NULL = 0)
 *   ids[t,j] = the expert with the j-th largest key; equal keys (+0 == -0)
 *              order by the lower expert id
 *   gates[t,j] = softmax of the RAW logits (the bias never enters the mix
 *              weights) over the k selected experts with MOE_F_RENORM, else
 *              over all E experts read at the selected ones.
 * logits fp32 [T,E] row-major; bias fp32 [E] or NULL; ids int32 [T,k];
 * gates fp32 [T,k].  All 4-byte aligned.  A NaN key sets MOE_ERR_DEVICE_NAN.
 */
moe_status_t moe_route(const moe_shape_t* shape, const float* logits, const float* bias,
                       int32_t* ids, float* gates, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/* Step 1 with rank-limited (node-limited) routing: each token's k experts
 * come from at most `max_ranks` of the R ranks ("19. All-to-all", opening
 * section: tokens limited to at most a few nodes so the slow hop stays
 * bounded; section "Why Qwen3.8's 512 experts is a systems statement":
 * node-limited routing as a constraint; "GPU MoE all-to-all", section "The
 * node boundary is the design decision").  The pages give no rank score; the
 * one used here is the largest key on the rank:
 *   score[r]  = max over the experts e of rank r of key[e]
 *   the max_ranks ranks with the largest scores are eligible (equal scores:
 *   the lower rank id); ids = the k largest keys among their experts (equal
 *   keys: the lower expert id); gates as moe_route.
 * 1 <= max_ranks; when max_ranks < R, k <= max_ranks * (E/R) is required
 * (else MOE_ERR_INVALID_ARG).  max_ranks >= R is exactly moe_route.  Same
 * buffers, layouts and errors as moe_route. */
moe_status_t moe_route_limited(const moe_shape_t* shape, const float* logits, const float* bias,
                               int32_t max_ranks, int32_t* ids, float* gates, void* ws,
                               size_t ws_bytes, moe_stream_t stream);

/* Remote-first, tile-aligned layout ("Mixture-of-experts acceleration
 * through overlap": a remote-owner-aligned layout where every tile belongs to
 * one destination rank and is written contiguously, and remote-first
 * scheduling: the data bound for other GPUs is produced first).  Same outputs
 * and rules as moe_layout, except that the rank slices are ordered as seen
 * from rank `home_rank` (the GPU holding the batch): home+1, home+2, ...
 * (mod R), and home's own slice last.  expert_off[e] is then the first row of
 * expert e (not increasing in e); rank_off[r] = expert_off[r*E/R] and
 * rank_off[R] = rows used.  With align = A (the grouped-GEMM tile height,
 * e.g. 128) every expert segment is a whole number of A-row tiles:
 *   tile_expert  int32 [N/A] expert owning rows i*A .. i*A+A-1, -1 past the
 *                rows used (NULL: not written)
 * 0 <= home_rank < R, else MOE_ERR_INVALID_ARG; home_rank = R-1 gives exactly
 * moe_layout.  The pages give no order among the remote slices; the rotation
 * is the usual all-to-all schedule. */
moe_status_t moe_layout_remote_first(const moe_shape_t* shape, const int32_t* ids,
                                     int32_t home_rank, int32_t* counts, int32_t* expert_off,
                                     int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                                     int32_t* src_idx, int32_t* tile_expert, void* ws,
                                     size_t ws_bytes, moe_stream_t stream);

/* The round-robin router, a diagnostic ("GPU MoE all-to-all", section "How
 * to tell whether the all-to-all is your bottleneck": replace the learned
 * router by a uniform round-robin assignment; a much faster exchange means
 * the problem is skew, not the wire):
 *   ids[t,j] = (t*k + j) mod E,  gates[t,j] = 1/k (rounded once to fp32)
 * k distinct experts per token; every expert gets T*k/E assignments when E
 * divides T*k.  Buffers as moe_route; no workspace. */
moe_status_t moe_route_round_robin(const moe_shape_t* shape, int32_t* ids, float* gates,
                                   moe_stream_t stream);

/* Aux-loss-free balancing: the per-expert bias update from a batch's
 * histogram ("19. All-to-all", section "Why the router can ruin your day":
 * a bias per expert bumped up or down based on recent load, used only for the
 * top-k decision).  For e in [0, E):
 *   bias[e] += gamma * sign(T*k/E - counts[e])
 * with the sign taken exactly in integers (an expert exactly at the mean
 * keeps its bias); one binary32 addition.  The pages give neither gamma nor
 * the form of the bump; this is the plainest reading.
 *   counts  int32 [E] assignments per expert (the counts moe_layout writes)
 *   bias    fp32 [E], updated in place (the bias moe_route takes next)
 * Both device buffers, 4-byte aligned; gamma finite and >= 0.  Runs on
 * `stream` after whatever wrote the counts; no workspace. */
moe_status_t moe_bias_update(const moe_shape_t* shape, const int32_t* counts, float gamma,
                             float* bias, moe_stream_t stream);

/* Steps 2 and 3 -- count histogram and layout scan ("GPU MoE all-to-all",
 * sections "Two collectives per layer" and "Bucketing"; "MoE All-to-All
 * Dispatch and Ragged Routing", section "Fixed Capacity vs. Ragged Routing").
 *   ids         int32 [T,k] expert ids (from moe_route or the caller)
 *   counts      int32 [E]   assignments per expert, before any drop
 *   expert_off  int32 [E+1] first row of each expert's segment; [E] = rows used
 *   rank_off    int32 [R+1] first row of each rank's slice; [R] = rows used
 *   rank_counts int32 [R]   rows of each rank's slice that hold a token -- the
 *                           per-destination counts an exchange posts first
 *   dst_pos     int32 [T,k] row of assignment (t,j); -1 if dropped
 *   src_idx     int32 [N]   t*k+j of the assignment in each row; -1 if empty
 * Within an expert, rows follow token order; in capacity mode the first C
 * assignments in that order are kept.  Results are deterministic: no output
 * depends on block scheduling.  An id outside [0,E) sets
 * MOE_ERR_DEVICE_RANGE and that assignment is treated as dropped.  A shape
 * with MOE_F_SRC_LAYOUT returns MOE_ERR_INVALID_ARG here and in the fused and
 * allocation-free layout calls (use moe_layout_src). */
moe_status_t moe_layout(const moe_shape_t* shape, const int32_t* ids, int32_t* counts,
                        int32_t* expert_off, int32_t* rank_off, int32_t* rank_counts,
                        int32_t* dst_pos, int32_t* src_idx, void* ws, size_t ws_bytes,
                        moe_stream_t stream);

/* Per-source-rank layout: the metadata and receive-side rows of a ragged
 * all-to-all ("GPU MoE all-to-all", sections "Two collectives per layer, and
 * what each one moves" -- counts before payload -- and "The message-size
 * distribution is the whole story" -- one message per (sender, receiver);
 * "MoE All-to-All Dispatch and Ragged Routing", section "Fixed Capacity vs.
 * Ragged Routing" -- per-sender-expert slots).  The shape must carry
 * MOE_F_SRC_LAYOUT; no page gives this interface.
 * The T tokens form R source shards of Ts = ceil(T/R) consecutive tokens
 * (shard s = tokens s*Ts .. s*Ts+Ts-1; trailing shards may be short or
 * empty).  Rows are ordered by destination rank r, then source shard s, then
 * expert e of rank r, then token order; segment (r, s, e) has index
 * i = (r*R + s)*(E/R) + e - r*(E/R) and holds round_up(count, align) rows
 * (dropless) or exactly C rows (capacity: the first C assignments of shard s
 * to expert e in token order are kept).
 *   ids          int32 [T,k]     expert ids
 *   src_counts   int32 [R,E]     assignments of shard s to expert e, before drops
 *   seg_off      int32 [R*E+1]   first row of segment i; [R*E] = rows used
 *   pair_counts  int32 [R,R]     [s][r] rows kept from shard s for rank r:
 *                                the size of the (s -> r) message
 *   rank_off     int32 [R+1]     first row of rank r's slice; [R] = rows used
 *   rank_counts  int32 [R]       rows kept for rank r from all shards
 *   dst_pos      int32 [T,k]     row of assignment (t,j); -1 if dropped
 *   src_idx      int32 [N]       t*k+j in each row; -1 if the row is empty
 * All caller-owned device buffers, 4-byte aligned.  The workspace is sized by
 * moe_workspace_bytes of the same shape.  Deterministic; an id outside [0,E)
 * sets MOE_ERR_DEVICE_RANGE and that assignment is dropped.  moe_dispatch
 * and moe_combine take the resulting dst_pos with the same shape. */
moe_status_t moe_layout_src(const moe_shape_t* shape, const int32_t* ids, int32_t* src_counts,
                            int32_t* seg_off, int32_t* pair_counts, int32_t* rank_off,
                            int32_t* rank_counts, int32_t* dst_pos, int32_t* src_idx, void* ws,
                            size_t ws_bytes, moe_stream_t stream);

/* Steps 1-3 in one launch: moe_route followed by moe_layout, fused so the
 * ids never leave the CTA that routed them before they are counted.  Same
 * arguments (the union of both calls), same results bit for bit, same error
 * behaviour. */
moe_status_t moe_route_layout(const moe_shape_t* shape, const float* logits, const float* bias,
                              int32_t* ids, float* gates, int32_t* counts, int32_t* expert_off,
                              int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                              int32_t* src_idx, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Step 4 -- dispatch ("GPU MoE all-to-all", sections "Bucketing" and
 * "Latency-bound at decode, bandwidth-bound at prefill").
 *   x       bf16 [T,H], 16-byte aligned
 *   dst_pos int32 [T,k] from moe_layout
 *   out     bf16 [N,H] (or e4m3 [N,H] with MOE_F_FP8), 16-byte aligned:
 *           row dst_pos[t,j] receives token t.  Rows no assignment maps to
 *           are not written.
 *   scales  fp32 [N,H/128] with MOE_F_FP8 (else ignored, may be NULL):
 *           per 128-channel block b of token t, amax = max|x|,
 *           scale = amax/448, codes = e4m3_rn_satfinite(x * (448/amax));
 *           amax == 0 gives codes 0 and scale 0.
 * A dst_pos value >= N sets MOE_ERR_DEVICE_RANGE and that copy is skipped. */
moe_status_t moe_dispatch(const moe_shape_t* shape, const void* x, const int32_t* dst_pos,
                          void* out, float* scales, void* ws, size_t ws_bytes,
                          moe_stream_t stream);

/* Steps 1-4 in one call: moe_route_layout followed by moe_dispatch, with the
 * same results bit for bit.  Inside this call the dispatch kernel starts
 * reading rows of x while the layout is still running (x is complete: every
 * kernel before this call has finished by then), so part of the copy overlaps
 * the latency-bound layout.  Arguments: the union of the two calls. */
moe_status_t moe_route_layout_dispatch(const moe_shape_t* shape, const float* logits,
                                       const float* bias, const void* x, int32_t* ids,
                                       float* gates, int32_t* counts, int32_t* expert_off,
                                       int32_t* rank_off, int32_t* rank_counts, int32_t* dst_pos,
                                       int32_t* src_idx, void* out, float* scales, void* ws,
                                       size_t ws_bytes, moe_stream_t stream);

/* Step 5 -- combine ("GPU MoE all-to-all", section "Two collectives per
 * layer": the inverse permutation scaled by the router's gate weights; "MoE
 * All-to-All Dispatch and Ragged Routing", section "Returning Tokens to the
 * Original GPU": the residual x + dx).
 *   out[t,c] = bf16_rn( sum_{j, dst_pos[t,j] >= 0} gates[t,j] * y[dst_pos[t,j], c]
 *                       + shared[t,c] + residual[t,c] )
 * accumulated in fp32 in slot order j = 0..k-1, then shared, then residual.
 *   y        bf16 [N,H] expert outputs in the layout's row order
 *   shared   bf16 [T,H] always-on expert output, or NULL
 *   residual bf16 [T,H] the layer input x, or NULL
 *   out      bf16 [T,H]
 * bf16 buffers 16-byte aligned.  A dropped slot contributes nothing; the other
 * gates are not rescaled. */
moe_status_t moe_combine(const moe_shape_t* shape, const void* y, const int32_t* dst_pos,
                         const float* gates, const void* shared, const void* residual,
                         void* out, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_layout without a workspace, for callers that cannot allocate device
 * memory: plugin or custom-op hosts that give a kernel only its inputs and
 * outputs, serving runtimes whose pool owns all device memory, and
 * latency-critical code that may not call cudaMalloc (it can synchronise the
 * device).  The pages have no counterpart to this call; it is an interface
 * convenience.
 *
 * Same arguments, results and determinism as moe_layout, minus `ws`.  The
 * scratch lives in a static device array of 256 + MOE_NOALLOC_TABLE_BYTES
 * bytes that every GPU loading the library keeps until the process exits.
 * Limit: the layout's two tile tables need 2 * min(ceil(T/16), 128) * E * 4
 * bytes, so min(ceil(T/16), 128) * E <= 65536 (any T for E <= 512, T <= 1024
 * for E = 1024); larger shapes return MOE_ERR_UNSUPPORTED and launch nothing.
 * Allocates nothing: no cudaMalloc / cudaFree or allocating library call.
 *  - Every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress), so an address never outlives its context (after
 *    cudaDeviceReset the array is loaded again, zero-filled).  The first call
 *    that sees an address on a device zero-fills the array there
 *    (cudaMemsetAsync on `stream`): make that first call before any stream
 *    capture.
 *  - Every call leaves the array ready for the next one; a call whose launch
 *    fails zero-fills it again.
 *  - All calls share the one array, so calls that overlap on the GPU race;
 *    order them (one stream, or events).
 *  - Device-side problems are not reported: the kernels record the first one
 *    in the array's error word, which no call reads or clears (an id outside
 *    [0,E) still comes out as dst_pos -1). */
#define MOE_NOALLOC_TABLE_BYTES (512u << 10)
moe_status_t moe_layout_noalloc(const moe_shape_t* shape, const int32_t* ids, int32_t* counts,
                                int32_t* expert_off, int32_t* rank_off, int32_t* rank_counts,
                                int32_t* dst_pos, int32_t* src_idx, moe_stream_t stream);

/* Self-test of the failure path of the kernels' bounded waits (the pages
 * have no counterpart): launches one warp that waits on an mbarrier no copy
 * will ever complete, with the same bounded wait the bulk-copy kernels use,
 * for timeout_us microseconds (1 .. 2000000).  When it gives up it records
 * MOE_ERR_DEVICE_TIMEOUT in the workspace header (detail = microseconds
 * waited) and returns; nothing stays in flight and the context stays usable.
 * Read the result with moe_get_device_error. */
moe_status_t moe_selftest_wait_timeout(void* ws, uint32_t timeout_us, moe_stream_t stream);

/* Synchronise `stream`, return the first device-side error recorded in `ws`
 * since the last read (MOE_OK if none) and clear it.  *detail (may be NULL)
 * receives the offending index (expert id, row, or block) when known. */
moe_status_t moe_get_device_error(void* ws, int32_t* detail, moe_stream_t stream);

/* Static description of a status code. */
const char* moe_status_string(moe_status_t status);

/* ABI version of this header (bumped on any incompatible change). */
#define MOE_ABI_VERSION 1
int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ROUTE07_H */
