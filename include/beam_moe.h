/*
 * beam_moe.h -- C ABI of the B200 (sm_100a) BEAM masked MoE-layer forward.
 *
 * The layer (BEAM article on aitrends.kr, "BEAM: Dynamic MoE 라우팅을 위한 Binary Expert
 * Activation Masking", four-step pipeline paragraph), per token x:
 *   Step 1  r = x W_r; keep the Top-K logits (set TK) and take a softmax over those K: g.
 *   Step 2  raw mask m_hat = sigmoid(x W_m).
 *   Step 3  m_i = 1 if m_hat_i >= 0.5 else 0, on the Top-K set only (evaluated as the mask
 *           logit (x W_m)_i >= 0, which is the same test in exact arithmetic).
 *   Step 4  g_hat = g (.) m, no renormalisation; y = sum_{i in TK, m_i = 1} g_hat_i E_i(x),
 *           plus the always-on shared experts (limitation (C) of the same article).
 * Experts whose mask is 0 are skipped: their weights are not read and none of their FLOPs
 * are spent (ai-feeds.com summary "BEAM: 用于 MoE 动态路由的二进制专家激活掩码", Method,
 * output and inference acceleration).  E_i is a SwiGLU FFN without biases:
 *   E(x) = W_d (silu(W_g x) * (W_u x)).
 * Optional segment routing ("Stepped MoE: Segment-Level Routing with Configurable Inference
 * Complexity", core method): with segment_len = S > 1, token t uses the Top-K set, gates and
 * mask of token S*floor(t/S); the experts still see x[t].
 *
 * Conventions for every call:
 *   - Pointers named *_dev are CUDA device pointers; *_host are host pointers.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - Calls return a beam_status_t; nothing throws.  beam_moe_last_error() gives a message for
 *     the last failing call on the calling thread.
 *   - A handle is not thread-safe: calls on one handle must not overlap.
 *   - Ties in the Top-K go to the lower expert index; Top-K outputs are in rank order.
 */
#ifndef BEAM_MOE_H
#define BEAM_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BEAM_OK = 0,
    BEAM_ERR_INVALID_ARG = 1,  /* a NULL pointer, a size out of range, an unsupported shape */
    BEAM_ERR_OOM = 2,          /* device allocation failed in beam_moe_create */
    BEAM_ERR_CUDA = 3,         /* a CUDA runtime error; the message has the CUDA error string */
    BEAM_ERR_UNSUPPORTED = 4,  /* valid request this build cannot serve (e.g. tensor path in fp32) */
    BEAM_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out; outputs are not valid */
    BEAM_ERR_NO_FORWARD = 6,   /* beam_moe_stats / get_routing before any forward */
    BEAM_ERR_RANGE = 7         /* bf16 layers: an fp16 intermediate of the last forward (H, or an
                                  expert output) overflowed; its y is not valid */
} beam_status_t;

enum { BEAM_DTYPE_F32 = 0, BEAM_DTYPE_BF16 = 1 };

/* forward flags */
#define BEAM_MASK_OFF     0x1u  /* plain Top-K: every Top-K slot kept (the W_m = 0 behaviour) */
#define BEAM_PATH_STREAM  0x2u  /* force the weight-streaming (GEMV) expert path */
#define BEAM_PATH_TENSOR  0x4u  /* force the tcgen05 tensor-core expert path (bf16 only) */
#define BEAM_NO_GRAPH     0x8u  /* launch the kernels directly instead of replaying a graph */
#define BEAM_FUSED_DECODE 0x10u /* batches of <= 32 tokens (bf16): one fused cooperative
                                   launch instead of separate kernels (opt-in; slower on B200) */
#define BEAM_TRAIN        0x20u /* training forward: every Top-K slot's expert is evaluated
                                   and the mask only scales the gates (g_hat = g * m), so that
                                   beam_moe_backward_router can follow (see there) */
#define BEAM_HOST_PIPELINE 0x40u /* beam_moe_forward_host only: run a batch of >= 1024 tokens
                                   as chunks whose copies overlap the forwards of the others
                                   (see beam_moe_forward_host) */
#define BEAM_HOST_Y_BF16  0x80u  /* beam_moe_forward_host only: y_host receives y rounded to
                                   bf16 (round to nearest even) instead of float32, half the
                                   device-to-host bytes; excludes BEAM_FUSED_DECODE (see
                                   beam_moe_forward_host) */
#define BEAM_HOST_ASYNC   0x100u /* beam_moe_forward_host only: return once the copies and the
                                   forward are queued, without waiting (see beam_moe_forward_host
                                   and beam_moe_host_wait) */
#define BEAM_Y_BF16       0x200u /* beam_moe_forward / _forward_routed: y is written as bf16
                                   (the float32 sum rounded to nearest even), T*D values at an
                                   8-byte aligned y; excludes BEAM_FUSED_DECODE (host calls use
                                   BEAM_HOST_Y_BF16) */

typedef struct {
    int32_t d_model;      /* D. bf16: multiple of 64; fp32: multiple of 4. <= 8192 (4096 fp32) */
    int32_t n_experts;    /* E routed experts, 1..256 */
    int32_t top_k;        /* K, 1..min(E, 32) */
    int32_t d_ff;         /* F, SwiGLU intermediate size per routed expert; multiple of 128 */
    int32_t n_shared;     /* S_sh always-on shared experts, 0..16 */
    int32_t d_ff_shared;  /* intermediate size per shared expert; multiple of 128 (0 if none) */
    int32_t dtype;        /* BEAM_DTYPE_F32 or BEAM_DTYPE_BF16: storage of x and all weights */
    int32_t segment_len;  /* 0 or 1: per-token routing; S > 1: segment routing */
    int32_t max_tokens;   /* largest T any forward will pass, 1..65536 */
} beam_moe_config_t;

/*
 * Layer weights, device pointers in the storage type, row-major:
 *   w_router [D][E]   r = x W_r            w_mask [D][E]   mask logits = x W_m
 *   w_gate   [E][F][D]  w_up [E][F][D]     w_down [E][D][F]
 *   ws_gate  [S][Fs][D] ws_up [S][Fs][D]   ws_down [S][D][Fs]  (NULL when n_shared == 0)
 * Borrowed only during beam_moe_create, which copies them into handle-owned layouts; the
 * caller may free its copies afterwards.
 */
typedef struct {
    const void *w_router, *w_mask;
    const void *w_gate, *w_up, *w_down;
    const void *ws_gate, *ws_up, *ws_down;
} beam_moe_weights_t;

/* Statistics of the last forward (BEAM article on aitrends.kr: Avg-K in the results
 * paragraph, L_reg = (1/K) sum_{i in TK} m_hat_i in the training paragraph, as means over
 * tokens). */
typedef struct {
    double avg_k;                /* mean number of kept experts per token */
    double l_reg;                /* mean over tokens of (1/K) sum_{i in TK} sigmoid(mask logit) */
    int32_t n_active_experts;    /* routed experts with at least one kept slot */
    int32_t n_tokens_all_masked; /* tokens whose Top-K slots were all masked */
    int32_t tokens;              /* T of the last forward */
    int32_t n_kept;              /* kept (token, slot) pairs = sum of per-expert counts */
} beam_moe_stats_t;

typedef struct beam_moe beam_moe_t;

/*
 * Build a layer handle: validates cfg, allocates every device buffer for up to
 * cfg->max_tokens tokens, and repacks the weights on `stream` (then synchronises it).
 * Returns BEAM_ERR_INVALID_ARG for a bad cfg/pointer, BEAM_ERR_OOM if allocation fails
 * (nothing is leaked), BEAM_ERR_CUDA otherwise on a CUDA error.  *out is set only on success.
 */
beam_status_t beam_moe_create(const beam_moe_config_t *cfg, const beam_moe_weights_t *w_dev,
                              void *stream, beam_moe_t **out);

/*
 * The hot path: y_dev[T][D] (float32) = BEAM layer of x_dev[T][D] (storage type), enqueued on
 * `stream` without any host synchronisation (per-expert token counts stay on the device).
 * Runs the fused router (x [W_r | W_m], Top-K, K-way softmax, mask, statistics), the
 * expert-grouping compaction, the grouped SwiGLU experts (kept experts only), the shared
 * experts and the fixed-order combine.  Deterministic: the same inputs give the same bits.
 * T = 0 is a no-op.  T > max_tokens or NULL pointers -> BEAM_ERR_INVALID_ARG.
 * flags: BEAM_MASK_OFF or BEAM_TRAIN (not both), and at most one of BEAM_PATH_STREAM /
 * BEAM_PATH_TENSOR (by default the path is chosen from T), BEAM_NO_GRAPH.  BEAM_TRAIN gives the
 * same y (up to rounding: masked slots add 0 * E_i(x)) at the cost of every Top-K expert; its
 * statistics count the mask (avg_k, l_reg, all-masked tokens) but n_active_experts, n_kept,
 * the counts and beam_moe_get_routing's keep / perm describe the evaluated slots (all of them).  x_dev and y_dev must stay valid until the stream
 * reaches the end of the call's work.
 * Replay: on a non-default stream that is not being captured, the first forward with a given
 * (x_dev, y_dev, T, flags) is captured into a CUDA graph owned by the handle, and later calls
 * with the same arguments replay it with one launch (one graph is kept; new arguments replace
 * it).  The contents of x_dev may change between calls; the pointers may not, for a replay.
 * BEAM_NO_GRAPH, the legacy default stream, an already-capturing stream and profiling all use
 * direct kernel launches.
 * BEAM_FUSED_DECODE: a bf16 forward of 1..32 tokens on the tensor-core path runs as one
 * cooperative launch of one block per SM (router, routing, compaction, both GEMMs, SwiGLU and
 * combine, separated by grid barriers) when the device supports cooperative launches; it is
 * launched directly, not replayed.  Without the flag the same forward runs as separate kernels
 * chained with programmatic dependent launch, which measured faster.
 */
beam_status_t beam_moe_forward(beam_moe_t *h, const void *x_dev, int32_t T, float *y_dev,
                               uint32_t flags, void *stream);

/*
 * beam_moe_forward with host buffers: copies x_host (T*D elements of the storage type) to a
 * handle-owned device buffer, runs the forward and copies y back to y_host (T*D float32, or
 * with BEAM_HOST_Y_BF16 T*D bf16: the combine stores y rounded to nearest even, as under
 * BEAM_Y_BF16, and the bf16 rows are copied; excludes BEAM_FUSED_DECODE), then synchronises
 * `stream`.  Pinned host memory gives full-bandwidth copies.
 * BEAM_HOST_PIPELINE (T >= 1024; flags may add BEAM_MASK_OFF, BEAM_PATH_*, BEAM_NO_GRAPH and
 * BEAM_HOST_Y_BF16):
 * the batch runs as 2 to 4 chunks of whole segments (about 1366 tokens each); chunk c's x copy,
 * forward and y copy are ordered on two copy streams and `stream`, so the copies of one chunk
 * overlap the forwards of its neighbours.  Each chunk is a complete forward of its tokens (the
 * same arithmetic per token; a token near a Top-K or mask tie may resolve differently from a
 * whole-batch forward, within the 1e-3 margin).  beam_moe_stats then describes the whole call
 * (statistics and counts added up over the chunks on the device); beam_moe_get_routing gives
 * topk_id, gate, mask_logit and keep of every token and returns BEAM_ERR_UNSUPPORTED if asked
 * for offsets, perm or inv (the compaction ran per chunk).  Direct launches (no graph replay).
 */
beam_status_t beam_moe_forward_host(beam_moe_t *h, const void *x_host, int32_t T, void *y_host,
                                    uint32_t flags, void *stream);

/*
 * BEAM_HOST_ASYNC (flags may add BEAM_MASK_OFF, BEAM_PATH_*, BEAM_NO_GRAPH, BEAM_HOST_Y_BF16):
 * beam_moe_forward_host queues the input copy, the whole-batch forward and the output copy and
 * returns without waiting.  Consecutive asynchronous calls on a handle alternate between two
 * handle-owned staging sets (the second is allocated by the first such call), so call k+1's
 * input copy and call k-1's output copy run while call k's forward does.  The forward runs on
 * `stream`, the copies on the handle's two copy streams, ordered by events.  x_host must stay
 * unchanged, and y_host unread, until beam_moe_host_wait returns.  beam_moe_stats and
 * beam_moe_get_routing describe the last call (they wait for its forward).  A later
 * synchronous host call waits for the asynchronous calls' copies first.
 *
 * beam_moe_host_wait: blocks until every queued host call's copies and the last forward are
 * done.
 */
beam_status_t beam_moe_host_wait(beam_moe_t *h);

/*
 * Statistics of the last forward; waits for it to finish.  counts_host, if not NULL,
 * receives the per-expert kept-slot counts (E int32).  Returns BEAM_ERR_TIMEOUT if a
 * bounded device wait of that forward ran out, and BEAM_ERR_RANGE if, in a bf16 layer, a value
 * the forward stored in fp16 (H = silu(W_g x) * (W_u x), or an expert's unsplit output) had a
 * magnitude of 65520 or more (it rounds to infinity) or was NaN: the kernels check every such
 * store and set a bit of the forward's error word, so an overflow is reported, not silent.
 */
beam_status_t beam_moe_stats(beam_moe_t *h, beam_moe_stats_t *out, int32_t *counts_host);

/*
 * Routing of the last forward, copied to host arrays (any may be NULL); waits for it:
 *   topk_id [T][K] int32 (rank order), gate [T][K] float32 (softmax over the K),
 *   mask_logit [T][K] float32, keep [T][K] uint8, offsets [E+1] int32 (exclusive prefix sum
 *   of per-expert counts), perm [n_kept] int32 (t*K+k of the kept pairs, by expert then
 *   token), inv [T][K] int32 (position in perm, or -1 for a masked slot).
 * A test and debugging hook; not needed by the forward.
 */
beam_status_t beam_moe_get_routing(beam_moe_t *h, int32_t *topk_id, float *gate,
                                   float *mask_logit, uint8_t *keep, int32_t *offsets,
                                   int32_t *perm, int32_t *inv);

/*
 * Per-stage timing for roofline reports.  beam_moe_profile_begin(h, n) makes the next (up to)
 * n forwards record a CUDA event pair around every kernel they launch (this disables the
 * launch overlap between kernels while it is on).  beam_moe_profile_end waits for them, adds
 * up the event times per stage into stage_ms[BEAM_N_STAGES] and the launches per stage into
 * stage_launches[BEAM_N_STAGES] (either may be NULL), sets *n_forwards, and switches timing
 * off.  beam_moe_stage_name(i) names stage i ("" when out of range).  On the tensor-core path
 * the shared experts' GEMMs run on a second stream, overlapping the routing; they are timed
 * under stages of their own (tc_shared_gateup, tc_shared_down), so that each stage's time
 * covers the work of one problem.  A fused decode forward is one launch, timed as the stage
 * fused_decode; the per-chunk statistics of a pipelined host call as chunk_stats.
 */
#define BEAM_N_STAGES 17
beam_status_t beam_moe_profile_begin(beam_moe_t *h, int32_t max_forwards);
beam_status_t beam_moe_profile_end(beam_moe_t *h, float *stage_ms, int32_t *stage_launches,
                                   int32_t *n_forwards);
const char *beam_moe_stage_name(int32_t stage);

/* Number of kernels the handle has launched since it was created (repacking excluded). */
int64_t beam_moe_launch_count(const beam_moe_t *h);

/*
 * Routing only, without allocating: Steps 1-3 (Top-K, K-way softmax, mask) for x_dev[T][D]
 * into caller-provided device arrays topk_id[T][K] int32, gate[T][K] f32, mask_logit[T][K]
 * f32, keep[T][K] uint8 and ghat[T][K] f32 (same values and layout as beam_moe_forward
 * produces; the 32-bit arrays 4-byte aligned, x 16-byte aligned), enqueued on `stream`.  The BEAM pages have no counterpart to this call; it exists
 * for callers that cannot allocate device memory when they route, e.g. a serving engine that
 * reserves all free device memory for its own pools up front, so any later cudaMalloc fails.
 * The call allocates nothing: its only scratch (the router logits and per-token statistics)
 * is a fixed array of BEAM_ROUTE_NOALLOC_SCRATCH_BYTES compiled into the library, which every
 * GPU that loads the library holds until the process exits.  It needs
 * ceil(ceil(T/S)*2E*4 / 256)*256 + 8*T bytes (S = segment length, 1 when off); a larger T is
 * rejected with BEAM_ERR_INVALID_ARG and a message giving both sizes.  The first call on
 * each device looks up the array's device address (cudaGetSymbolAddress) and caches it; make
 * that first call before any stream capture.  Later calls on a stream that is not capturing
 * look it up again (so a reset context that reloaded the library's module is served); calls
 * during a capture use the cached address.  All calls share the array and it keeps the last
 * call's contents, so calls whose GPU work overlaps (different streams or threads) race on it
 * and must be serialised by the caller.  flags: 0 or BEAM_MASK_OFF.  The handle's own buffers,
 * statistics, launch count and profile are untouched (its weights are only read), so the call
 * may be enqueued between forwards; like every call on a handle it must not run concurrently
 * with another call on the same handle from a second host thread.
 */
#define BEAM_ROUTE_NOALLOC_SCRATCH_BYTES (2u << 20)
beam_status_t beam_moe_route_noalloc(beam_moe_t *h, const void *x_dev, int32_t T,
                                     int32_t *topk_id, float *gate, float *mask_logit,
                                     uint8_t *keep, float *ghat, uint32_t flags, void *stream);

/*
 * Self-test of the library's bounded device waits (no counterpart on the BEAM pages): runs one
 * tiny kernel whose thread waits on an mbarrier that nothing completes, giving up after
 * timeout_us microseconds (1..2,000,000).  The kernel then records the expiry and returns
 * normally, so the context stays usable.  Returns BEAM_ERR_TIMEOUT when the wait expired as
 * designed (the expected outcome); BEAM_ERR_INVALID_ARG for a bad timeout; BEAM_ERR_CUDA
 * otherwise.  Synchronises `stream`.  Every wait in the forward's kernels uses the same
 * primitive, with a limit of 2 s.
 */
beam_status_t beam_moe_wait_selftest(int32_t timeout_us, void *stream);

/*
 * ---------------------------------------------------------------- cross-layer routing
 * The mask generator of "Stepped MoE: Segment-Level Routing with Configurable Inference
 * Complexity" (core method and its inference paragraph): one pass over the output z of the
 * model's dense prefix gives the routing logits of every MoE layer at once, one decision per
 * segment of S tokens taken at the segment's first token, so that every layer's experts are
 * known before the first MoE layer runs (and their weights can be fetched ahead).
 * Combined with BEAM, layer l's decision is BEAM's Steps 1-3 with that layer's generator
 * weights: r = z W_r^(l), mask logits z W_m^(l); Top-K of r (ties to the lower index), a
 * softmax over the K, keep = mask logit >= 0 on the Top-K set, g_hat = g * keep.  The logits of
 * all layers come from one GEMM, z_leaders [W_r^(1) | W_m^(1) | ... | W_r^(L) | W_m^(L)].
 */
typedef struct beam_gen beam_gen_t;

typedef struct {
    int32_t d_model;      /* D of z; same rules as beam_moe_config_t.d_model */
    int32_t n_layers;     /* L, 1..512 */
    int32_t n_experts;    /* E per layer, 1..256 */
    int32_t top_k;        /* K, 1..min(E, 32) */
    int32_t dtype;        /* BEAM_DTYPE_F32 or BEAM_DTYPE_BF16: storage of z and the weights */
    int32_t segment_len;  /* 0 or 1: one decision per token; S > 1: per segment of S tokens */
    int32_t max_tokens;   /* largest T any call will pass, 1..65536 */
} beam_gen_config_t;

/*
 * Routing of L layers (or of one layer: every pointer offset to that layer), device arrays,
 * layer-major:
 *   topk_id [L][T][K] int32 (rank order)   gate [L][T][K] f32 (softmax over the K)
 *   mask_logit [L][T][K] f32               keep [L][T][K] uint8
 *   ghat [L][T][K] f32 (gate * keep)       n_keep [L][T] int32 (kept slots per token)
 *   lreg [L][T] f32 ((1/K) sum_{TK} sigmoid(mask logit))
 *   active [L][(E+31)/32] uint32: bit e%32 of word e/32 of layer l is set when some token of
 *          the call keeps expert e in layer l (the experts whose weights that layer will read)
 * A token of segment s carries the decision of the segment's first token, S*s.
 */
typedef struct {
    int32_t *topk_id;
    float *gate;
    float *mask_logit;
    uint8_t *keep;
    float *ghat;
    int32_t *n_keep;
    float *lreg;
    uint32_t *active;
} beam_routing_t;

/*
 * Build a mask generator from w_router_dev[L][D][E] and w_mask_dev[L][D][E] (device, storage
 * type, row-major per layer; borrowed during the call only: they are repacked into one
 * [L*2E][D] matrix owned by the handle), on `stream` (then synchronised).  Errors as for
 * beam_moe_create.
 */
beam_status_t beam_gen_create(const beam_gen_config_t *cfg, const void *w_router_dev,
                              const void *w_mask_dev, void *stream, beam_gen_t **out);

/*
 * Routing of every layer for z_dev[T][D]: every array of *out except `active` (which may be
 * NULL) must hold L*T*K (or L*T) elements; enqueued on `stream` without synchronising.  bf16
 * generators with d_model a multiple of 64 compute the logits on the tensor cores (tcgen05),
 * others with a CUDA-core GEMV; then one warp per (segment, layer) takes the decision.
 * flags: 0 or BEAM_MASK_OFF (every Top-K slot kept).  T = 0 is a no-op.  z must be 16-byte
 * aligned and the 32-bit arrays 4-byte aligned (else BEAM_ERR_INVALID_ARG).  A bounded device
 * wait that ran out is reported by beam_gen_sync (BEAM_ERR_TIMEOUT).
 */
beam_status_t beam_gen_route(beam_gen_t *g, const void *z_dev, int32_t T,
                             const beam_routing_t *out, uint32_t flags, void *stream);

/* Wait for the generator's last call; BEAM_ERR_TIMEOUT if one of its bounded waits ran out. */
beam_status_t beam_gen_sync(beam_gen_t *g);

/* Free the generator's device buffers (waits for its pending work).  NULL is ignored. */
void beam_gen_destroy(beam_gen_t *g);

/*
 * beam_moe_forward with the routing given instead of computed: r points at one layer's
 * topk_id, keep, ghat, n_keep and lreg (required; gate and mask_logit optional, only kept for
 * beam_moe_get_routing; active unused), e.g. layer l's slice of a beam_gen_route output.  The
 * forward skips the router and the Top-K/mask step and runs the compaction, the experts, the
 * shared experts and the combine exactly as beam_moe_forward does; beam_moe_stats then
 * describes the given routing.  flags: BEAM_PATH_STREAM / BEAM_PATH_TENSOR / BEAM_NO_GRAPH
 * (BEAM_MASK_OFF and BEAM_FUSED_DECODE are rejected: the mask is part of the routing).  The
 * graph replay key includes the routing pointers.  The routing arrays must stay valid until
 * the stream reaches the end of the call's work, and, for beam_moe_get_routing, until that
 * call.  Alignment: topk_id 4 bytes (16 when top_k is 4, 8 or 16), keep top_k bytes when
 * top_k is 4, 8 or 16, ghat / n_keep / lreg 4 bytes.
 */
beam_status_t beam_moe_forward_routed(beam_moe_t *h, const void *x_dev, int32_t T,
                                      const beam_routing_t *r, float *y_dev, uint32_t flags,
                                      void *stream);

/*
 * ---------------------------------------------------------------- training: routing gradient
 * The gradient of the routing under BEAM's training recipe (BEAM article on aitrends.kr,
 * training paragraph: L = L_lm + alpha L_bal + beta L_reg, L_reg = (1/K) sum_{i in TK}
 * |m_hat_i|, the straight-through estimator carrying the binary mask's gradient to m_hat;
 * ai-feeds.com summary, Method, binarisation and straight-through estimator).  With
 * dy = dL/dy, for token t and Top-K slot k (expert i, gate g_k, mask logit l_k, m_k = l_k >= 0):
 *   s_tk = <dy_t, E_i(x_t)>  (= dL/dg_hat),   dL/dg_k = s_tk m_k,
 *   dL/dm_hat_k = s_tk g_k + reg_scale / (T K)       (straight through: dm/dm_hat = 1; L_reg
 *                                                     the mean over tokens of the per-token term)
 *   d_mask_logit_k = dL/dm_hat_k sigmoid(l_k) (1 - sigmoid(l_k))
 *   d_gate_logit_k = g_k (dL/dg_k - sum_j g_j dL/dg_j)   (softmax over the K; logits outside
 *                                                     the Top-K get nothing)
 *   dW_r[d][i] = sum_t x_t[d] d_gate_logit_tk,  dW_m[d][i] = sum_t x_t[d] d_mask_logit_tk,
 *   dx_t = sum_k d_gate_logit_tk W_r[:, i] + d_mask_logit_tk W_m[:, i]   (the routing's share
 *          of dL/dx; the experts' own backward is not part of this call).
 * With segment routing the segment's tokens share their first token's decision: their terms
 * are summed at that token, which alone gets logit gradients and a nonzero dx row.  L_bal is
 * not defined on the pages and has no term here.
 *
 * Precondition: the handle's last forward was a beam_moe_forward with BEAM_TRAIN (flags may
 * add BEAM_PATH_* / BEAM_NO_GRAPH; not BEAM_MASK_OFF or BEAM_FUSED_DECODE) on the same x_dev
 * contents and the same T, and no forward ran since (else BEAM_ERR_NO_FORWARD).  That forward
 * evaluated every Top-K slot's expert and kept the outputs in the handle.
 * Arguments (device pointers, enqueued on `stream`, no host synchronisation):
 *   x_dev [T][D] storage type (16-byte aligned), dy_dev [T][D] float32 (16-byte aligned),
 *   reg_scale = dL/dL_reg (beta), dw_router_dev / dw_mask_dev [D][E] float32 (overwritten),
 *   dx_dev [T][D] float32 (overwritten, 16-byte aligned); d_gate_logit_dev,
 *   d_mask_logit_dev and dghat_dev [T][K] float32 are optional outputs (NULL to skip) holding
 *   the per-slot gradients above (0 at the tokens of a segment after its first) and s.
 * Every sum runs in a fixed order: the same inputs give the same bits.  T = 0 is a no-op.
 * The call allocates nothing: its workspace was allocated with the handle.
 */
beam_status_t beam_moe_backward_router(beam_moe_t *h, const void *x_dev, const float *dy_dev,
                                       int32_t T, float reg_scale, float *dw_router_dev,
                                       float *dw_mask_dev, float *dx_dev,
                                       float *d_gate_logit_dev, float *d_mask_logit_dev,
                                       float *dghat_dev, void *stream);

/*
 * ---------------------------------------------------------------- expert parallelism
 * The BEAM article on aitrends.kr names multi-GPU interaction as future work (limitation (D)).
 * Here the routed experts are split over P ranks in contiguous blocks (beam_ep_expert_range:
 * rank q holds experts [floor(qE/P), floor((q+1)E/P))); every rank routes its own tokens over
 * all E experts and runs the shared experts itself.  One forward of a rank's batch:
 *   1. beam_moe_ep_dispatch on the rank's routing handle: Steps 1-3 and the compaction.  X_perm
 *      (the kept rows, sorted by expert and then token) stays on the device; the rows for rank
 *      q's experts are the contiguous range given by the per-expert counts.
 *   2. the caller exchanges the counts of each rank's experts and the rows (all-to-all);
 *   3. each rank turns the rows it received into one-slot tokens (beam_ep_recv_routing) and runs
 *      its expert handle (an ordinary handle over its E_local experts with top_k = 1 and no
 *      shared experts) with beam_moe_forward_routed: the compaction groups the rows by expert,
 *      the grouped GEMMs run, and y holds each row's expert output in the received order;
 *   4. the caller sends those rows back (the reverse all-to-all): the rank gets its own rows'
 *      expert outputs in X_perm order;
 *   5. beam_moe_ep_combine: y = sum over the token's kept slots in rank order of g_hat Y + the
 *      shared experts (the same fixed order as beam_moe_forward, so the result is deterministic).
 * dynamic_expert_routing_b200/ep.py drives the exchange with torch.distributed (NCCL).
 */

/*
 * A routing-only handle: as beam_moe_create, but w_gate / w_up / w_down are ignored (may be
 * NULL) and no routed expert weights are held.  It routes over cfg->n_experts experts and runs
 * the shared experts; beam_moe_forward / _routed / backward_router on it give
 * BEAM_ERR_UNSUPPORTED.  beam_moe_stats and beam_moe_get_routing describe its last dispatch.
 */
beam_status_t beam_moe_create_ep(const beam_moe_config_t *cfg, const beam_moe_weights_t *w_dev,
                                 void *stream, beam_moe_t **out);

/*
 * Steps 1-3, the compaction and the shared experts for x_dev[T][D] on `stream`, without host
 * synchronisation.  xperm_dev (caller-owned device buffer of T*K rows of D elements in the
 * storage type, 16-byte aligned) receives X_perm: its first n_kept rows are the kept rows,
 * sorted by expert and then token; counts_dev [E] int32 (device) the kept rows per expert.
 * flags: BEAM_MASK_OFF, BEAM_PATH_STREAM or BEAM_PATH_TENSOR (the path of the shared experts).
 * Works on any handle.  The shared experts' output and the dispatch's gates stay in the handle
 * for beam_moe_ep_combine.
 */
beam_status_t beam_moe_ep_dispatch(beam_moe_t *h, const void *x_dev, int32_t T, uint32_t flags,
                                   void *xperm_dev, int32_t *counts_dev, void *stream);

/*
 * y_dev[T][D] float32 of the last dispatch: the fixed-order combine of y_perm_dev [n_kept][D]
 * float32 (the expert outputs of the dispatched rows, in X_perm order; 16-byte aligned) with
 * the dispatch's gates, plus the shared experts.  BEAM_ERR_NO_FORWARD before any dispatch.
 */
beam_status_t beam_moe_ep_combine(beam_moe_t *h, const float *y_perm_dev, float *y_dev,
                                  void *stream);

/* Host only: the experts of rank q of P, [*first, *first + *count), for E experts. */
beam_status_t beam_ep_expert_range(int32_t E, int32_t P, int32_t q, int32_t *first,
                                   int32_t *count);

/*
 * The routing of the n_rows rows an expert rank received, as one-slot tokens: source s sent
 * recv_counts_dev[s][e] rows (device, [P][E_local] int32) of local expert e, source-major and
 * expert-minor; n_rows must be their sum.  Writes topk_id [n_rows] int32 (the local expert),
 * keep [n_rows] uint8 (1), ghat [n_rows] float32 (1), n_keep [n_rows] int32 (1) and lreg
 * [n_rows] float32 (0), device arrays (4-byte aligned), for beam_moe_forward_routed of the
 * expert handle.  P * E_local <= 4096.
 */
beam_status_t beam_ep_recv_routing(const int32_t *recv_counts_dev, int32_t P, int32_t E_local,
                                   int32_t n_rows, int32_t *topk_id_dev, uint8_t *keep_dev,
                                   float *ghat_dev, int32_t *n_keep_dev, float *lreg_dev,
                                   void *stream);

/*
 * ---------------------------------------------------------------- training: SoftTopK
 * The differentiable top-k of "Stepped MoE: Segment-Level Routing with Configurable Inference
 * Complexity" (its SoftTopK entry and core method): the routing logits pass through a continuous
 * relaxation of the top-k indicator, so the choice of experts trains end to end, while the
 * layers use the {0,1} top-k mask.  The page names the relaxation but gives no formula; the one
 * used is the limited-multi-label projection (Amos, Xu and Kolter, "The Limited Multi-Label
 * Projection Layer", 2019), for logits r of one row, 1 <= K <= E and temperature tau > 0:
 *   y_i = sigmoid((r_i - nu) / tau),  nu such that sum_i y_i = K
 * (y = 1 everywhere when K = E).  As tau -> 0, y tends to the top-k indicator.
 * beam_softtopk_forward: logits_dev [T][E] float32 -> y_dev [T][E] float32, and optionally
 *   mask_dev [T][E] uint8 (the hard Top-K indicator, ties to the lower index, as the layer's
 *   router) and nu_dev [T] float32.  nu is found by safeguarded Newton iteration in float32
 *   (bisection inside the sign bracket whenever a step leaves it) until a step is below
 *   2^-16 tau; y agrees with a float64 solution to about 1e-5.
 * beam_softtopk_backward: dlogits_dev [T][E] = the Jacobian of y (through nu) applied to
 *   dy_dev [T][E]: with h_i = y_i (1 - y_i) / tau,
 *   dlogits_j = h_j (dy_j - sum_i h_i dy_i / sum_i h_i)   (0 when sum_i h_i = 0);
 *   y_dev is the forward's y.  Used as the straight-through gradient of the hard mask, or as the
 *   exact gradient of the relaxation.
 * Device pointers, row-major, 4-byte aligned; E <= 256; enqueued on `stream` without host
 * synchronisation; T = 0 is a no-op.  Bad sizes, tau <= 0 or NULL pointers give
 * BEAM_ERR_INVALID_ARG.  Deterministic (fixed reduction order).
 */
beam_status_t beam_softtopk_forward(const float *logits_dev, int32_t T, int32_t E, int32_t K,
                                    float tau, float *y_dev, uint8_t *mask_dev, float *nu_dev,
                                    void *stream);
beam_status_t beam_softtopk_backward(const float *y_dev, const float *dy_dev, int32_t T,
                                     int32_t E, float tau, float *dlogits_dev, void *stream);

/* Free every device buffer of the handle (waits for its pending work).  NULL is ignored. */
void beam_moe_destroy(beam_moe_t *h);

/* Message of the last failing call on this thread ("" if none). */
const char *beam_moe_last_error(void);

/* Library version string. */
const char *beam_moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BEAM_MOE_H */
