/*
 * kvpop.h -- C ABI of the KVpop fixed-budget KV cache, decode-time hot path.
 *
 * Method: "KVpop -- Key-Value Cache Compression with Predictive Online
 * Pruning" (summary page of arXiv 2607.05061v2).  Every KV head keeps a
 * bounded cache of budget B = S + W + K tokens, the same for every head:
 * S attention-sink tokens, a protected window of the W most recent tokens,
 * and K long-range slots holding the running top-k of the tokens that have
 * left the window, ranked by a small headwise scorer on [k; v]
 * (page §3 "Fixed-budget pruning", §C.1 "Mask Definition", §E.1-§E.2,
 * §I "KVpop Pseudocode").  Optional delayed scoring (page §3 "Stateful
 * scorers", §E.4 "Delayed Readout") is a D-slot staging ring between the
 * window and the long-range slots: a token is scored D steps after it leaves
 * the window.  Staged tokens stay cached and are attended.
 *
 * Conventions for every call:
 *  - Return value: KVPOP_OK (0) or a negative KVPOP_ERR_* code.  Nothing
 *    throws or aborts across the ABI.  Arguments are validated before any
 *    work is enqueued; a call that fails validation enqueues nothing.
 *  - Device pointers point to memory on the device the handle was created on.
 *    The library never allocates or frees device memory: the caller owns all
 *    of it and lends it for the duration of the call (inputs) or the handle's
 *    lifetime (the cache buffer).
 *  - Work is asynchronous on the caller's CUDA stream (`stream`, a
 *    cudaStream_t; NULL = legacy default stream).  Only kvpop_create,
 *    kvpop_inspect and kvpop_get_error synchronise.
 *  - Calls on one handle must be ordered on one stream (or by the caller's
 *    events): the handle's split-K scratch is shared by its layers.
 *  - All batch rows share one sequence length.  Layers are independent and
 *    each keeps its own position counter (on the device).
 *  - Element type of q, k, v, the cache and the output: config.dtype.
 *    Scores are fp32 (the page, §F, ranks and selects in float32).
 */
#ifndef KVPOP_H
#define KVPOP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define KVPOP_OK 0
#define KVPOP_ERR_INVALID_ARG -1      /* null pointer, out-of-range layer, bad flag */
#define KVPOP_ERR_BAD_SHAPE -2        /* shape combination not valid / not built */
#define KVPOP_ERR_ORDER -3            /* call out of order (e.g. prefill after decode) */
#define KVPOP_ERR_CONTEXT_OVERFLOW -4 /* position counter would pass max_context */
#define KVPOP_ERR_CUDA -5             /* a CUDA runtime call failed */
#define KVPOP_ERR_DEVICE -6           /* a kernel recorded an error (see kvpop_get_error) */
#define KVPOP_ERR_TIMEOUT -7          /* a bounded device-side wait gave up */
#define KVPOP_ERR_SCRATCH_LIMIT -8    /* needs more scratch than kvpop_decode_step_noalloc's static buffer */

/* Size of the static split-K scratch buffer behind kvpop_decode_step_noalloc
 * (16 MiB on every GPU that loads the library, held until the process exits). */
#define KVPOP_NOALLOC_SCRATCH_BYTES (16u << 20)

/* Element types. */
#define KVPOP_DTYPE_F32 0
#define KVPOP_DTYPE_BF16 1

/* Scorer kinds (kvpop_config.scorer_kind). */
#define KVPOP_SCORER_MLP 0    /* stateless MLP, or the linear scorer when scorer_hidden = 0 (page §E.2) */
#define KVPOP_SCORER_MLSTM 1  /* stateful mLSTM scorer with delayed readout (page §A, §E.3, §E.4) */

/* Floats of one (layer, KV head) block of kvpop_config.mlstm_w: rows of 2d
 * weights W_q (p rows), W_k (p), W_v (dv), w_i, w_f, then w_o (dv), b_i, b_f,
 * b_o, padded to a multiple of 4. */
#define KVPOP_MLSTM_HEAD_FLOATS(p, dv, d) ((2 * (p) + (dv) + 2) * 2 * (d) + (((dv) + 3 + 3) / 4) * 4)

/* Flags. */
#define KVPOP_FLAG_EXTERNAL_SCORES 1u /* caller supplies every token's score instead of the MLP */
#define KVPOP_FLAG_DEBUG_CHECKS 2u    /* kernels check slot bookkeeping and NaN scores */

/* Device error bits reported by kvpop_get_error. */
#define KVPOP_DEVERR_CONTEXT_OVERFLOW 1
#define KVPOP_DEVERR_TIMEOUT 2
#define KVPOP_DEVERR_BAD_INDEX 4
#define KVPOP_DEVERR_NAN_SCORE 8
#define KVPOP_DEVERR_STATE_MISMATCH 16

typedef struct kvpop_config {
  int32_t batch;        /* batch rows b >= 1 */
  int32_t n_layers;     /* layers L >= 1 */
  int32_t n_q_heads;    /* query heads Hq, a multiple of n_kv_heads (GQA) */
  int32_t n_kv_heads;   /* KV heads Hkv >= 1 */
  int32_t head_dim;     /* d: 64 or 128 (bf16), 64 (fp32) */
  int32_t sinks;        /* S >= 0 */
  int32_t window;       /* W >= 1 */
  int32_t topk;         /* K >= 0 long-range slots; budget B = S + W + K */
  int32_t delay;        /* D >= 0 staging slots for delayed scoring (outside B) */
  int32_t ref_context;  /* prompt length the compression ratio is quoted against; 0 = no check */
  float compression_ratio; /* redundant, checked: |(1 - CR) * ref_context - B| <= 0.5 */
  int32_t max_context;  /* positions must stay below this (int32 positions) */
  int32_t max_prefill_chunk; /* largest n_tokens of one kvpop_prefill call */
  int32_t dtype;        /* KVPOP_DTYPE_F32 or KVPOP_DTYPE_BF16 */
  int32_t scorer_hidden; /* MLP 2d -> hidden -> 1 with hidden in {32, 64, 128}, or 0 = linear scorer */
  /* Scorer weights, device fp32, borrowed for the handle's lifetime
   * (may be NULL with KVPOP_FLAG_EXTERNAL_SCORES):
   *   w1 [L][Hkv][hidden][2d]  (input x = [k; v], page §E.1)
   *   b1 [L][Hkv][hidden], w2 [L][Hkv][hidden], b2 [L][Hkv]
   * score = w2 . relu(W1 x + b1) + b2 (page §E.2, stateless MLP scorer).
   * With scorer_hidden = 0 (page §E.2, stateless headwise linear scorer):
   * w1 [L][Hkv][2d] and b2 [L][Hkv], score = w1 . x + b2; b1, w2 may be NULL. */
  const float* w1;
  const float* b1;
  const float* w2;
  const float* b2;
  uint32_t flags;       /* KVPOP_FLAG_* */
  /* Optional temporal decay (page §B.3 "Temporal Decay and Static
   * Priorities"): device fp32 [L][Hkv] holding ln(gamma_h), each finite and
   * <= 0 (0 < gamma_h <= 1), borrowed for the handle's lifetime; NULL = no
   * decay.  Token j becomes eligible at step e_j = j + W + D; its effective
   * score at step q is s_j + (q - e_j) ln gamma_h, which ranks like the
   * static priority p_j = s_j - e_j ln gamma_h.  The library ranks by p_j,
   * formed once in fp32 (one rounding, like fmaf), and stores p_j as the
   * long-range slots' scores.  Requires max_context <= 2^24. */
  const float* log_decay;
  /* Scorer kind: KVPOP_SCORER_MLP (w1/b1/w2/b2 above) or KVPOP_SCORER_MLSTM
   * (the fields below; w1/b1/w2/b2 and scorer_hidden are then unused).  The
   * mLSTM scorer (page §A "Background: Linear Attention and mLSTM", §E.3
   * "mLSTM Scorer", §E.4 "Delayed Readout"): per KV head a recurrent state
   * (matrix memory C [2p][dv], normaliser n [2p], stabiliser m) in fp64 in
   * the cache buffer, updated by every token t with x_t = [k_t; v_t]:
   *   phi_t = [softmax(W_k x_t); softmax(-W_k x_t)] (Hedgehog feature map),
   *   i~ = w_i . x_t + b_i, log f = log sigmoid(w_f . x_t + b_f),
   *   m' = max(log f + m, i~), C' = e^(log f + m - m') C + e^(i~ - m') phi_t (W_v x_t)^T,
   *   n' = e^(log f + m - m') n + e^(i~ - m') phi_t;
   * the token u that becomes eligible at step q = u + W + D is read out from
   * the state after token q with r = Hedgehog(W_q x_u):
   *   h = C^T r / max(|n . r|, e^-m),  score = w_o . SiLU(h) + b_o,
   * rounded once to fp32.  Each decode step updates the state with the new
   * token before deciding the boundary token, so the decision is taken in
   * the step itself (one extra small launch per layer and step).  The
   * prefill attention calls do not take this scorer (KVPOP_ERR_BAD_SHAPE). */
  int32_t scorer_kind;
  int32_t mlstm_p;        /* Hedgehog projection size p, 1..16 (2p features) */
  int32_t mlstm_dv;       /* value size dv, 1..32 */
  const float* mlstm_w;   /* device fp32 [L][Hkv][KVPOP_MLSTM_HEAD_FLOATS(p, dv, d)], 16-byte aligned,
                             borrowed for the handle's lifetime (may be NULL with KVPOP_FLAG_EXTERNAL_SCORES) */
} kvpop_config;

typedef struct kvpop_handle kvpop_handle;

/* Offsets (bytes, from dev_mem) of the cache arrays, for inspection and tests.
 * Layer l's arrays start at offset + l * *_layer_stride. */
typedef struct kvpop_layout_info {
  size_t kv_offset, kv_layer_stride;       /* [units][slots][2][d] (key row, value row) */
  size_t pos_offset, pos_layer_stride;     /* int32 [units][slots], -1 = empty */
  size_t score_offset, score_layer_stride; /* fp32 [units][slots] */
  size_t state_offset, state_layer_stride; /* int32 [units][4] = {n_seen, n_topk, 0, 0} */
  int32_t slots_per_unit;                  /* S + W + D + K */
  int32_t units;                           /* batch * n_kv_heads; unit = b * Hkv + h */
  int32_t row_bytes;                       /* 2 * d * sizeof(dtype) */
  int32_t topk_base;                       /* first long-range slot, S + W + D */
} kvpop_layout_info;

/* Device bytes the caller must allocate for `cfg` (cache, slot metadata,
 * split-K and prefill scratch).  Validates cfg.  Host only.
 * Page §3 "Fixed-budget pruning" and §C.1 "Mask Definition": every KV head
 * keeps at most B = S + W + K tokens, the same budget for every head, so the
 * cache of a layer is units x (S + W + D + K) slots, fixed at creation
 * (D = the staging ring of delayed scoring, §E.4).  The pages quote
 * compression ratios (75%, 88%) without a formula; this library reads them
 * as CR = 1 - B / ref_context and checks cfg.compression_ratio against it.
 * Errors: KVPOP_ERR_INVALID_ARG (null argument; bad dtype, flag or scorer
 * pointer; compression ratio out of [0, 1) or not matching the budget),
 * KVPOP_ERR_BAD_SHAPE (shape outside the supported set). */
int kvpop_cache_bytes(const kvpop_config* cfg, size_t* bytes);

/* Binds a caller-allocated device buffer (>= kvpop_cache_bytes, 256-byte
 * aligned, on the current device) and initialises it (empty cache,
 * synchronously).  The buffer must outlive the handle.  *out receives the
 * handle (host memory owned by the library until kvpop_destroy).
 * Page §3 "Fixed-budget pruning" (a hard, fixed-size cache: eviction is
 * permanent, so the cache never grows past its budget) and §C.1 (the budget
 * is reached once the sequence is long enough; until then every slot that
 * holds a token is attended).  Errors: KVPOP_ERR_INVALID_ARG (null, short or
 * misaligned buffer, buffer not device memory), KVPOP_ERR_BAD_SHAPE (cfg
 * outside the supported shapes), KVPOP_ERR_CUDA (a CUDA call failed); *out
 * is NULL then. */
int kvpop_create(const kvpop_config* cfg, void* dev_mem, size_t bytes, kvpop_handle** out);

/* Page §I "KVpop Pseudocode" (score every KV entry, keep the sinks, the
 * recent window and the running-prefix top-k of the eligible tokens) and
 * §C.1 "Mask Definition", applied to a whole prompt chunk at once.
 * Appends a chunk of n_tokens prompt tokens to layer `layer` (positions
 * n_seen .. n_seen + n_tokens - 1).  k, v: device [b][Hkv][n_tokens][d].
 * ext_scores: device fp32 [b][Hkv][n_tokens] (required with
 * KVPOP_FLAG_EXTERNAL_SCORES, ignored otherwise).  After the call the layer
 * holds the running prefix top-k state at its last token (page §I): the
 * long-range slots keep the K best eligible tokens; survivors keep their
 * slots and admitted tokens fill free/vacated slots in ascending order.
 * Must precede the layer's first decode step (else KVPOP_ERR_ORDER);
 * 0 <= n_tokens <= max_prefill_chunk.  Errors (nothing enqueued):
 * KVPOP_ERR_INVALID_ARG (bad handle or layer, negative n_tokens, null k or v,
 * missing ext_scores), KVPOP_ERR_BAD_SHAPE (n_tokens > max_prefill_chunk),
 * KVPOP_ERR_ORDER, KVPOP_ERR_CONTEXT_OVERFLOW (positions would reach
 * max_context); KVPOP_ERR_CUDA if a launch fails. */
int kvpop_prefill(kvpop_handle* h, int32_t layer, const void* k, const void* v, int32_t n_tokens,
                  const float* ext_scores, void* stream);

/* One decode step of one layer for all batch rows: page §3 "Fixed-budget
 * pruning" (sinks + protected window + running top-k, eviction permanent),
 * §C.1 "Mask Definition" (during decoding attention runs directly over the
 * retained cache entries), §E.4 "Delayed Readout" (the token u = q - w
 * becomes eligible at q; with the staging ring, D steps later) and §I
 * "KVpop Pseudocode" (the running prefix top-k rule).  With p = the layer's
 * position counter:
 *  1. window append and boundary update: the token leaving the window (after
 *     D staging steps when D > 0) is scored by the MLP on [k; v] (or its
 *     caller score) and replaces the minimum of the long-range set only if
 *     its key (score, -position) is strictly larger; while the long-range set
 *     is not full it takes the next free slot; the new token's k/v is written
 *     to its window slot;
 *  2. GQA attention of the new queries over all occupied slots (softmax,
 *     scale 1/sqrt(d), fp32 accumulation).
 * q: device [b][Hq][d]; k_new, v_new: device [b][Hkv][d]; out: device
 * [b][Hq][d] (same element type); ext_score: device fp32 [b][Hkv], the score
 * of the token being appended (required with KVPOP_FLAG_EXTERNAL_SCORES).
 * q, k_new, v_new and out must be 16-byte aligned (KVPOP_ERR_INVALID_ARG
 * otherwise).  The position counter then advances by one.  Errors (nothing
 * enqueued): KVPOP_ERR_INVALID_ARG (bad handle or layer, null or misaligned
 * pointer, missing ext_score), KVPOP_ERR_CONTEXT_OVERFLOW (the position
 * counter has reached max_context), KVPOP_ERR_BAD_SHAPE; KVPOP_ERR_CUDA if
 * the launch fails.  Device-side failures (a bounded wait that gave up,
 * debug-check mismatches) are reported later by kvpop_get_error. */
int kvpop_decode_step(kvpop_handle* h, int32_t layer, const void* q, const void* k_new, const void* v_new,
                      void* out, const float* ext_score, void* stream);

/* kvpop_decode_step for callers that cannot allocate device memory.
 * The KVpop pages have no counterpart: this is a deployment variant.
 *
 * Who needs it: code that runs where nobody may call cudaMalloc -- a plugin
 * inside a serving engine whose memory planner owns every device byte and
 * hands the plugin only the tensors it planned, or a latency-critical decode
 * loop that must not risk the device-wide synchronisation a cudaMalloc or
 * cudaFree can cause.  This call allocates nothing and calls no allocating
 * routine.  Its split-K partials and arrival tickets live in one static
 * device buffer that is part of the library image
 * (KVPOP_NOALLOC_SCRATCH_BYTES per GPU), not in the handle's buffer; the
 * handle's own split-K region is left untouched.
 *
 * Arguments, results and errors are those of kvpop_decode_step, plus:
 *  - KVPOP_ERR_SCRATCH_LIMIT (nothing enqueued) when the handle needs more
 *    scratch than the static buffer holds.  The need is
 *    units * 64 * G * (head_dim + 2) * 4 bytes plus units * 4, each part
 *    rounded up to 256 bytes (units = batch * n_kv_heads, G = n_q_heads /
 *    n_kv_heads); with G = 4, head_dim = 128 that is up to 126 units.
 *  - KVPOP_ERR_INVALID_ARG when the current device is not the handle's.
 *  - Set-up: the first call on a device (with that device current) looks up
 *    the buffer's device address once and keeps it for the process; make
 *    that first call before any stream capture begins.
 *  - Every call on a device shares the one buffer, which keeps what the last
 *    call left there.  The call clears the arrival tickets (the only part
 *    that must start at zero) on `stream` before its kernel; the partials
 *    are always written before they are read.  Calls whose work overlaps on
 *    the GPU (other streams, other handles, other host threads) race on the
 *    buffer and give wrong results: order them on one stream or by events. */
int kvpop_decode_step_noalloc(kvpop_handle* h, int32_t layer, const void* q, const void* k_new,
                              const void* v_new, void* out, const float* ext_score, void* stream);

/* The two halves of kvpop_decode_step (same passages: page §3, §C.1, §E.4,
 * §I), for callers that schedule them apart
 * (same arguments and semantics; append must precede attend for each step).
 * kvpop_decode_append: step 1 only (window append, boundary scoring and
 * argmin-replace); advances the position counter.
 * kvpop_decode_attend: step 2 only, over the cache as it stands (the query of
 * the token appended last).  Calling attend again without an append repeats
 * the same attention. */
int kvpop_decode_append(kvpop_handle* h, int32_t layer, const void* k_new, const void* v_new,
                        const float* ext_score, void* stream);
int kvpop_decode_attend(kvpop_handle* h, int32_t layer, const void* q, void* out, void* stream);

/* Parallel sparse prefill attention (page §C "Efficient Running Top-k Sparse
 * Attention": §C.1 Mask Definition, §C.2 Fenwick-Tree Cutoff Computation).
 * Computes, for every position q of a prompt of n_tokens tokens (positions
 * 0 .. n_tokens - 1) and every query head, the attention output under the
 * fixed-budget mask: q attends to exactly the set a decode step at q would
 * attend to -- the sinks, the recent W + D positions (its own included) and
 * the running top-k of the tokens eligible at q (scored as kvpop_prefill
 * scores them, decay included) -- with softmax scale 1/sqrt(d) and fp32
 * accumulation.  Does not read or change the cache or its position counter;
 * any layer's scorer weights may be used at any time.
 *
 * Running cutoffs: with m = q - W - D, token j (S <= j <= n_tokens-1-W-D)
 * is in the long-range set exactly for m in [j, c_j); c_j = INT32_MAX when j
 * is still kept at the last position, c_j = j when it is never admitted.
 * Tokens that never become eligible in the prompt get -1.
 *
 * q: device [b][Hq][n_tokens][d]; k, v: device [b][Hkv][n_tokens][d];
 * out: device [b][Hq][n_tokens][d] (config.dtype); lse: device fp32
 * [b][Hq][n_tokens] receiving each row's natural-log softmax normaliser
 * log sum_j exp(q.k_j / sqrt(d)), or NULL; ext_scores: device fp32
 * [b][Hkv][n_tokens] (required with KVPOP_FLAG_EXTERNAL_SCORES, ignored
 * otherwise).  q, k, v, out and workspace must be 16-byte aligned, lse 4-byte
 * aligned.
 * workspace: caller-owned device scratch of at least
 * kvpop_prefill_attention_workspace_bytes(n_tokens) bytes; after the call its
 * first units * n_tokens int32 hold the cutoffs c_j ([units][n_tokens]).
 * Errors: KVPOP_ERR_INVALID_ARG (null or misaligned pointer, workspace too
 * small, bad layer), KVPOP_ERR_BAD_SHAPE (G not dividing 64, head_dim other
 * than 64/128, S + K + W + D + P above 16384 where P = 64/G for fp32 and
 * 256/G for bf16, more than 65535 units, the mLSTM scorer),
 * KVPOP_ERR_CONTEXT_OVERFLOW (n_tokens > max_context); nothing is enqueued
 * then.  n_tokens = 0 is a no-op. */
int kvpop_prefill_attention_workspace_bytes(const kvpop_handle* h, int32_t n_tokens, size_t* bytes);
int kvpop_prefill_attention(kvpop_handle* h, int32_t layer, const void* q, const void* k, const void* v,
                            int32_t n_tokens, const float* ext_scores, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream);

/* The attention stage of kvpop_prefill_attention alone, from the running
 * cutoffs that a previous kvpop_prefill_attention call of the same prompt
 * (same layer's scorer, same k, v and n_tokens) left in `workspace`: the
 * prompt is not scored again and the cutoffs are not recomputed (page §C.2:
 * the cutoffs are computed once and the mask is evaluated from them on the
 * fly).  For a caller that runs several query sets over one prompt's mask.
 * The result equals that call's bit for bit when q, k and v are the same.
 * Arguments, layouts and errors as kvpop_prefill_attention (no ext_scores);
 * the workspace contents are the caller's responsibility. */
int kvpop_prefill_attention_from_cutoffs(kvpop_handle* h, int32_t layer, const void* q, const void* k, const void* v,
                                         int32_t n_tokens, void* out, float* lse, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* kvpop_prefill and kvpop_prefill_attention in one call, for a whole prompt
 * on an empty layer: the prompt is scored once, its attention outputs (and
 * log-normalisers, if lse is not NULL) are computed under the running top-k
 * mask, and the layer's cache is built from the same scores and cutoffs --
 * the long-range slots receive the tokens whose cutoff is INT32_MAX (kept at
 * the last position) in ascending position order, exactly what kvpop_prefill
 * of the whole prompt as one chunk places.  Afterwards the layer is ready for
 * decode steps (position counter n_tokens).  Arguments, layouts, workspace
 * and errors as kvpop_prefill_attention, plus KVPOP_ERR_ORDER when the layer
 * has seen any token.  Page §C.1 / §C.2 (mask and cutoffs) and §I (running
 * prefix top-k). */
int kvpop_prefill_with_attention(kvpop_handle* h, int32_t layer, const void* q, const void* k, const void* v,
                                 int32_t n_tokens, const float* ext_scores, void* out, float* lse, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Copies layer `layer`'s slot -> position map (int32 [units][slots]), slot
 * scores (fp32 [units][slots]) and per-unit state (int32 [units][4]) to HOST
 * buffers; any of them may be NULL.  Synchronises `stream`.  Test and
 * diagnostic call; no passage of the pages defines it.  Errors:
 * KVPOP_ERR_INVALID_ARG (bad handle or layer), KVPOP_ERR_CUDA. */
int kvpop_inspect(kvpop_handle* h, int32_t layer, int32_t* pos_out, float* score_out, int32_t* state_out,
                  void* stream);

/* Fills *out with the layout of the device buffer.  Diagnostic call; no
 * passage of the pages defines it.  KVPOP_ERR_INVALID_ARG on a null argument. */
int kvpop_get_layout(const kvpop_handle* h, kvpop_layout_info* out);

/* Failure reporting of this library (no passage of the pages defines it).
 * Synchronises the device and reads the device error word.  Returns KVPOP_OK
 * if no kernel recorded an error, KVPOP_ERR_CONTEXT_OVERFLOW / _TIMEOUT /
 * _DEVICE otherwise (device_bits, if not NULL, receives the KVPOP_DEVERR_*
 * bits), or KVPOP_ERR_CUDA if the device reported an asynchronous error. */
int kvpop_get_error(kvpop_handle* h, int32_t* device_bits);

/* Clears the device error word (asynchronously, on `stream`).  Failure
 * reporting of this library; no passage of the pages defines it. */
int kvpop_clear_error(kvpop_handle* h, void* stream);

/* Test hook (no passage of the pages defines it): ORs `bits` into the device
 * error word on `stream`, so host-side failure handling can be exercised
 * without making any kernel fail. */
int kvpop_debug_poison_error(kvpop_handle* h, int32_t bits, void* stream);

/* Test hook (no passage of the pages defines it), honoured only by builds of
 * this library compiled with KVPOP_TEST_HOOKS, which also shorten the decode
 * kernel's merge-queue waits; other builds return KVPOP_ERR_INVALID_ARG and
 * change nothing.  hook = 1: in every later decode step, one consumer warp
 * finishes its work but never reports that it is done, so its CTA's merge
 * helpers wait until their bound runs out and the error word records
 * KVPOP_DEVERR_TIMEOUT (the kernel still returns; no copy is in flight
 * during that wait).  hook = 0 turns it off. */
int kvpop_debug_set_hook(kvpop_handle* h, int32_t hook);

/* Releases the handle's host state.  Does not touch the device buffer.
 * Resource management of this library; no passage of the pages defines it.
 * KVPOP_ERR_INVALID_ARG on NULL. */
int kvpop_destroy(kvpop_handle* h);

/* Static description of a status code (diagnostic; no passage defines it). */
const char* kvpop_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KVPOP_H */
