/*
 * hymba.h — C ABI of the B200 (sm_100a) Hymba hybrid-head layer forward.
 *
 * The layer is the fused hybrid-head module of "Hymba: A Hybrid-head
 * Architecture for Small Language Models" (arXiv 2411.13676), §2.1 Eq. (1)-(3):
 * one input projection feeds an attention branch (Eq. 1) and a Mamba SSM
 * branch (Eq. 2) in parallel; each branch is RMS-normalised, re-scaled per
 * channel by beta, the two are averaged and projected back (Eq. 3).  Meta
 * tokens are prepended to the input (§2.3 Eq. 4); sliding-window layers use the
 * "A-shape" mask that always sees the meta tokens, a few layers are global, and
 * consecutive sliding-window layers share K/V (§2.2; authors' OpenReview reply
 * "Cache Optimization" / "Meta Tokens").
 *
 * Conventions for every entry point:
 *   - Positions index X~ = [R; X]: rows 0..n_meta-1 are the meta tokens, then the
 *     real tokens.  A sequence has L = n_meta + n_tokens rows.
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *     densely packed, with the layouts stated below.  The library never frees,
 *     copies or retains them beyond the call, except that a layer handle keeps
 *     the weight pointers given to hymba_layer_create until destroy.
 *   - Storage dtype HYMBA_BF16: activations, K/V, conv state and the W_in, W_x,
 *     W_out matrices are bf16 (accumulation in fp32); HYMBA_F32: all fp32.
 *     Per-channel parameters, W_dt and the SSM state are always fp32.
 *   - Compute calls are asynchronous on `stream`; they do not allocate, do not
 *     synchronise and never abort.  Every argument is validated on the host
 *     before anything is launched; a failed check launches nothing and returns
 *     an error code (hymba_last_error() gives a one-line reason).  Device-side
 *     faults and bounded-wait timeouts surface through hymba_stream_status().
 *   - Device pointers and leading dimensions must be 16-byte aligned (TMA).
 */
#ifndef HYMBA_H_
#define HYMBA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HYMBA_API __attribute__((visibility("default")))
#else
#define HYMBA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *hymba_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  HYMBA_OK = 0,
  HYMBA_ERR_INVALID_ARG = 1,  /* bad shape, null pointer, misaligned pointer   */
  HYMBA_ERR_UNSUPPORTED = 2,  /* valid request the library does not implement */
  HYMBA_ERR_WORKSPACE = 3,    /* workspace smaller than the query returned     */
  HYMBA_ERR_NOT_BOUND = 4,    /* K/V sharing: consumer/producer mismatch       */
  HYMBA_ERR_CUDA = 5,         /* a CUDA runtime call failed                    */
  HYMBA_ERR_TIMEOUT = 6,      /* a device-side bounded wait gave up            */
  HYMBA_ERR_DEVICE = 7        /* no usable sm_100 device                       */
} hymba_status;

typedef enum { HYMBA_F32 = 0, HYMBA_BF16 = 1 } hymba_dtype;

/* Layer configuration: shape, attention layout and storage dtype.
 * Appendix E Table 11 (1.5B): d_model 1600, n_heads 25, n_kv_heads 5 ("query
 * groups"), d_state 16, window 1024; n_meta 128 (OpenReview reply on meta-token
 * count).  head_dim_v must equal d_inner / n_heads so the two branches have the
 * same width in Eq. (3).  dt_rank is the rank of W_delta = W_dt W_x[:dt_rank]
 * (Mamba's low-rank delta). */
typedef struct {
  int d_model;       /* d                                              */
  int n_heads;       /* H query heads                                  */
  int n_kv_heads;    /* Hkv; H % Hkv == 0; head h reads kv head h/(H/Hkv) */
  int head_dim_qk;   /* d_qk (64)                                      */
  int head_dim_v;    /* d_v = d_inner / n_heads                        */
  int d_inner;       /* E, SSM channels                                */
  int d_state;       /* N (16)                                         */
  int d_conv;        /* K, causal depthwise conv width (4)             */
  int dt_rank;       /* R                                              */
  int n_meta;        /* m meta tokens prepended to every sequence      */
  int window;        /* W: key j visible from query i iff i - j < W or j < m (sliding-window layers) */
  int is_global;     /* 1: full causal attention (window ignored)      */
  hymba_dtype dtype;
  float rms_eps;     /* eps of the per-branch RMS norm                 */
  float softmax_scale; /* 0 -> 1/sqrt(head_dim_qk) (OpenReview reply Q2) */
  float rope_base;   /* rotary position embedding of Q and K (§2.5 changes "the RoPE base";
                        no value is given): 0 = none; > 1: pair (2i, 2i+1) of every head
                        turned by p * rope_base^(-2i/head_dim_qk) at X~ position p, applied
                        by the input projection (head_dim_qk a power of two).  Layers that
                        share K/V must use the same base. */
  int branch_chunks; /* the two branches side by side (Fig. 1 and §2.1: the attention and
                        SSM heads read the same input in parallel; the OpenReview reply on
                        speed proposes two CUDA streams).  0 or 1: every step of a prefill
                        runs in order on the caller's stream.  n in 2..8: the prefill splits
                        the batch into min(n, batch) chunks; each chunk's selective scan runs
                        on the handle's own low-priority side stream, beside the next chunk's
                        projections and attention (raised priority), and the caller's stream
                        waits for it before that chunk's fusion.  The results are the same
                        bits as the serial order.  The side stream and its events belong to
                        the handle (created with it, on the device current at creation), so
                        a handle with n >= 2 takes its prefill and decode calls from one host
                        thread at a time.  A decode step of such a handle runs its SSM branch
                        on the side stream beside the attention (same bits as in order). */
} hymba_layer_config;

/* Weights of one layer (device pointers, kept by the handle, never copied).
 * P = H*d_qk + Hkv*(d_qk + d_v) + 2E for a layer that owns its K/V, and
 * P = H*d_qk + 2E for a K/V-sharing consumer (no K/V rows).  Row order of W_in
 * follows W_in_proj = [W^Q, W^K, W^V, W^SSM, W^G] (§2.1). */
typedef struct {
  const void  *w_in;      /* [P, d_model]                 dtype  */
  const float *conv_w;    /* [d_inner, d_conv]; tap d_conv-1 multiplies the current row */
  const float *conv_b;    /* [d_inner]                           */
  const void  *w_x;       /* [dt_rank + 2*d_state, d_inner] dtype; rows: delta_r, B, C */
  const float *w_dt;      /* [d_inner, dt_rank] fp32 (dt_rank % 4 == 0) */
  const float *b_dt;      /* [d_inner]                           */
  const float *a_log;     /* [d_inner, d_state]; A = -exp(a_log) */
  const float *d_skip;    /* [d_inner] D                          */
  const float *beta_attn; /* [d_inner] beta_1                     */
  const float *beta_ssm;  /* [d_inner] beta_2                     */
  const void  *w_out;     /* [d_model, d_inner]           dtype  */
} hymba_layer_weights;

typedef struct hymba_layer hymba_layer; /* opaque host handle */

/* Full-length K/V of one prefill: k [batch, L, Hkv*d_qk], v [batch, L, Hkv*d_v]
 * (token-major, as the input projection produces them).  A layer that owns its
 * K/V writes them and stamps `owner`, `batch`, `rows`; a consumer bound with
 * hymba_kv_share_bind reads them in place and checks the stamp. */
typedef struct {
  void *k;
  void *v;
  int batch;
  int rows;
  uint64_t owner;   /* set by the library; 0 = never written */
} hymba_kv_seq;

/* Decode K/V store of a layer that owns K/V: k [batch, Hkv, capacity, d_qk],
 * v [batch, Hkv, capacity, d_v].  Slot of position p: p for meta rows
 * (p < m) and for every row of a global layer; m + (p - m) mod W for real rows
 * of a sliding-window layer, so capacity >= m + W (window) or >= the largest
 * position + 1 (global).  `owner` as in hymba_kv_seq. */
typedef struct {
  void *k;
  void *v;
  int batch;
  int capacity;
  uint64_t owner;
} hymba_kv_cache;

/* Recurrent state of the SSM branch: h [batch, d_inner, d_state] fp32 and the
 * last d_conv-1 rows of the SSM input x_ssm, conv [batch, d_conv-1, d_inner]
 * (dtype; oldest row first). */
typedef struct {
  float *h;
  void *conv;
} hymba_ssm_cache;

/* ---- handles ------------------------------------------------------------ */

/* Validates the configuration, records it and the weight pointers.  No device
 * work.  Returns INVALID_ARG / UNSUPPORTED with a reason on failure. */
HYMBA_API hymba_status hymba_layer_create(const hymba_layer_config *cfg, const hymba_layer_weights *w,
                                hymba_layer **out);
HYMBA_API void hymba_layer_destroy(hymba_layer *layer);
/* 1 if this handle reads another layer's K/V. */
HYMBA_API int hymba_layer_is_consumer(const hymba_layer *layer);

/* Cross-layer K/V sharing (§2.2 "Cross-layer KV sharing"): `consumer` stops
 * projecting K/V (its W_in must have no K/V rows) and attends over the K/V
 * written by `producer`.  Host only.  Checks that n_kv_heads, head dims,
 * n_meta, window and is_global match, that the producer is not itself a
 * consumer, and that the consumer's W_in width is the consumer width;
 * returns NOT_BOUND / INVALID_ARG otherwise.  Binding twice rebinds. */
HYMBA_API hymba_status hymba_kv_share_bind(hymba_layer *consumer, const hymba_layer *producer);

/* ---- prefill ------------------------------------------------------------ */

/* Bytes of device workspace hymba_layer_prefill needs for this batch/length. */
HYMBA_API hymba_status hymba_layer_prefill_workspace(const hymba_layer *layer, int batch, int n_tokens,
                                           size_t *bytes);

/* Byte offsets inside the prefill workspace of the intermediates left there by
 * the last prefill (row-major, M = batch*L rows).  For stage-by-stage checks. */
typedef struct {
  size_t q;       /* [M, H*d_qk]          dtype */
  size_t x_ssm;   /* [M, E]               dtype */
  size_t gate;    /* [M, E] SiLU(z)       dtype */
  size_t u;       /* [M, E] conv+SiLU     dtype */
  size_t xdbl;    /* [M, R+2N] fp32: delta_r, B, C */
  size_t delta;   /* [M, E] softplus      dtype */
  size_t y_ssm;   /* [M, E] gated scan    dtype */
  size_t o_attn;  /* [M, E] attention     dtype */
  size_t fused;   /* [M, E] Eq. 3 inside W_out(.)  dtype */
  size_t rope;    /* [L, d_qk/2] (cos, sin) fp32 pairs of the rotary embedding (if any) */
  size_t sched;   /* [64] uint32 work counters of the persistent kernels (zeroed by each
                     prefill; each launch of the call takes one) */
  size_t total;
} hymba_prefill_layout;
HYMBA_API hymba_status hymba_layer_prefill_layout(const hymba_layer *layer, int batch, int n_tokens,
                                        hymba_prefill_layout *out);

/* One layer over `batch` sequences of L = n_meta + n_tokens rows: the hybrid-head
 * module of §2.1 (Eq. 3 over the attention heads of Eq. 1 and the SSM heads of Eq. 2)
 * on X~ = [R; X] (§2.3 Eq. 4), with the A-shape or global mask of §2.2 and, for a
 * bound consumer, the producer's K/V ("Cross-layer KV sharing", §2.2).
 *   x   [batch, L, d_model] dtype : X~ (meta rows included; the caller builds
 *                                   [R; X] for the first layer, later layers
 *                                   take the previous layer's output as is)
 *   y   [batch, L, d_model] dtype : Y of Eq. (3) for every row
 *   kv  full-length K/V: written by a layer that owns K/V (required), read by a
 *       consumer (must carry its producer's stamp and the same batch/rows)
 *   kv_cache  optional (NULL): a K/V owner also writes its decode store — the
 *       meta rows and the rows of the last W positions (all rows if global);
 *       other slots are left untouched.  Must be NULL for a consumer.
 *   ssm_cache optional (NULL): final SSM state h_L and the last d_conv-1 x_ssm rows.
 *   workspace >= hymba_layer_prefill_workspace() bytes, 256-byte aligned. */
HYMBA_API hymba_status hymba_layer_prefill(hymba_layer *layer, int batch, int n_tokens,
                                 const void *x, void *y, hymba_kv_seq *kv,
                                 hymba_kv_cache *kv_cache, hymba_ssm_cache *ssm_cache,
                                 void *workspace, size_t workspace_bytes, hymba_stream_t stream);

/* ---- meta-token cache --------------------------------------------------- */

/* The meta tokens are the same rows at the head of every sequence (§2.3 Eq. 4), so
 * their part of a layer's work does not depend on the input: the paper notes that it can
 * be done offline, the meta tokens acting as a learned initialisation of the K/V cache
 * and the SSM state (§2.3, "Initialization for KV cache and SSM state").  A meta cache
 * holds that part for one layer, computed once (batch 1):
 *   k, v  [n_meta, Hkv*d_qk] / [n_meta, Hkv*d_v] dtype: the meta rows' K/V (a layer that
 *         owns its K/V; unused for a consumer, which reads its producer's)
 *   h     [d_inner, d_state] fp32: the SSM state after the meta rows
 *   conv  [d_conv-1, d_inner] dtype: the last d_conv-1 x_ssm rows of the meta rows
 *   y     [n_meta, d_model] dtype: the layer's output for the meta rows, which is the
 *         next layer's meta input
 *   owner set by hymba_layer_meta_precompute (0 = not computed).
 * Device buffers owned by the caller, 16-byte aligned. */
typedef struct {
  void *k;
  void *v;
  float *h;
  void *conv;
  void *y;
  uint64_t owner;
} hymba_meta_cache;

/* Workspace bytes of hymba_layer_meta_precompute (a batch-1 prefill of the meta rows). */
HYMBA_API hymba_status hymba_layer_meta_workspace(const hymba_layer *layer, size_t *bytes);

/* Fills `meta` for this layer from x_meta [n_meta, d_model] dtype: the meta tokens R
 * for the first layer, the previous layer's meta->y for later ones.  A consumer passes
 * its producer's meta cache (stamp checked, NOT_BOUND otherwise); a K/V owner passes
 * NULL.  Asynchronous on `stream`; INVALID_ARG if the layer has no meta tokens. */
HYMBA_API hymba_status hymba_layer_meta_precompute(hymba_layer *layer, const void *x_meta,
                                                   hymba_meta_cache *meta,
                                                   const hymba_meta_cache *producer_meta,
                                                   void *workspace, size_t workspace_bytes,
                                                   hymba_stream_t stream);

/* Workspace bytes of hymba_layer_prefill_cached (intermediates of the real rows only). */
HYMBA_API hymba_status hymba_layer_prefill_cached_workspace(const hymba_layer *layer, int batch,
                                                            int n_tokens, size_t *bytes);

/* hymba_layer_prefill for the real rows only, starting from this layer's meta cache:
 *   x, y  [batch, n_tokens, d_model] dtype: the real rows of X~ (positions n_meta..L-1)
 *         and their outputs (the meta rows' outputs are meta->y, the same for every
 *         sequence)
 *   meta  computed by hymba_layer_meta_precompute for this layer (NOT_BOUND otherwise)
 *   kv    full-length K/V as for hymba_layer_prefill (L = n_meta + n_tokens rows per
 *         sequence): a K/V owner copies its meta rows' K/V into rows 0..n_meta-1 of each
 *         sequence and writes rows n_meta..L-1; a consumer reads its producer's.
 *   kv_cache, ssm_cache, workspace as for hymba_layer_prefill (ssm_cache receives the
 *         state after the whole sequence).
 * Same results as hymba_layer_prefill on X~ = [R; X] for rows n_meta..L-1, with the
 * meta rows' work done once instead of once per sequence.  n_tokens >= 1. */
HYMBA_API hymba_status hymba_layer_prefill_cached(hymba_layer *layer, int batch, int n_tokens,
                                                  const void *x, void *y, const hymba_meta_cache *meta,
                                                  hymba_kv_seq *kv, hymba_kv_cache *kv_cache,
                                                  hymba_ssm_cache *ssm_cache, void *workspace,
                                                  size_t workspace_bytes, hymba_stream_t stream);

/* ---- decode ------------------------------------------------------------- */

/* Bytes of device workspace hymba_layer_decode_step needs for positions up to max_pos. */
HYMBA_API hymba_status hymba_layer_decode_workspace(const hymba_layer *layer, int batch, int64_t max_pos,
                                                    size_t *bytes);

/* One new token per sequence at X~ position `pos` (same for every sequence;
 * pos >= n_meta): the same module for a single row, reading the layer's caches — the
 * meta rows plus the sliding window of K/V, or every row for a global layer (§2.2, §2.3
 * "learned cache initialization"), and the constant-size SSM state of Eq. 2's
 * recurrence (§2.1).  x_t, y_t [batch, d_model] dtype.
 *   kv_cache: a K/V owner appends this token's K/V at its slot and attends over
 *     its own store; a consumer attends over its producer's store (stamp
 *     checked), which the producer must have updated for this position first.
 *   ssm_cache: read and updated in place (h and the conv window).
 * A sliding-window layer attends over positions {0..m-1} and
 * {max(m, pos-W+1)..pos}; a global layer over 0..pos. */
HYMBA_API hymba_status hymba_layer_decode_step(hymba_layer *layer, int batch, int64_t pos,
                                     const void *x_t, void *y_t, hymba_kv_cache *kv_cache,
                                     hymba_ssm_cache *ssm_cache, void *workspace,
                                     size_t workspace_bytes, hymba_stream_t stream);

/* Decode step that allocates nothing and takes no workspace argument.
 *
 * For callers that cannot call cudaMalloc: code whose device memory is all
 * carved up in advance by another owner (an inference server's memory pool,
 * an engine's arena) and that has no way to ask it for a workspace, or a
 * latency-critical loop that must not pay for cudaMalloc's implicit device
 * synchronisation.  This entry point has no counterpart on the paper's pages.
 *
 * It runs exactly hymba_layer_decode_step (same arguments, same results) with
 * its scratch in a buffer of HYMBA_DECODE_STATIC_SCRATCH_BYTES that the
 * library holds in device memory of every GPU that loads it, until exit.
 * A request needing more scratch than that (hymba_layer_decode_workspace) is
 * rejected with HYMBA_ERR_WORKSPACE before anything is launched; 40 MiB covers
 * a batch of 128 on a sliding-window layer of the 1.5B shape (m + W = 1152).
 * The first call on a device looks up the buffer's device address (with that
 * device current), and so does the first call after that device's context has been
 * torn down and created again; make such a first call before any stream capture.  All calls
 * share the one buffer, which keeps the last call's contents (the step zeroes
 * what it accumulates into): calls that may overlap on the GPU race, so issue
 * them in order on one stream. */
#define HYMBA_DECODE_STATIC_SCRATCH_BYTES (40u << 20)
HYMBA_API hymba_status hymba_layer_decode_step_static(hymba_layer *layer, int batch, int64_t pos,
                                                      const void *x_t, void *y_t,
                                                      hymba_kv_cache *kv_cache,
                                                      hymba_ssm_cache *ssm_cache,
                                                      hymba_stream_t stream);

/* ---- the Hymba block ------------------------------------------------------ */

/* A block of the model (Fig. 4 (b); Appendix E Table 11: MLP hidden 5504 at 1.5B): the
 * hybrid-head module and an MLP, each behind an RMS norm with a learnable weight and
 * inside a residual:
 *     h = x + M(norm1(x)),   out = h + W_down (SiLU(W_gate n) * (W_up n)),  n = norm2(h)
 * (the pages give the caption and the MLP width only; this gated form is the one whose
 * parameter count gives the printed 1.52B).  The mixer M is the layer of `layer` (its
 * weights, K/V sharing, caches and RoPE as for hymba_layer_prefill / _decode_step).
 *   norm1, norm2  [d_model] fp32
 *   w_gate_up     [2 * mlp_hidden, d_model] dtype: row 2i is W_gate's row i, row 2i+1 W_up's
 *   w_down        [d_model, mlp_hidden] dtype
 * mlp_hidden a multiple of 8.  Device pointers, 16-byte aligned, owned by the caller. */
typedef struct {
  const float *norm1;
  const float *norm2;
  const void *w_gate_up;
  const void *w_down;
  int mlp_hidden;
} hymba_block_weights;

HYMBA_API hymba_status hymba_block_prefill_workspace(const hymba_layer *layer, int mlp_hidden, int batch,
                                                     int n_tokens, size_t *bytes);
/* The block over `batch` sequences of L = n_meta + n_tokens rows of the residual stream:
 * x, y [batch, L, d_model] dtype (distinct buffers); other arguments as for
 * hymba_layer_prefill.  A stack of blocks chains y into the next block's x. */
HYMBA_API hymba_status hymba_block_prefill(hymba_layer *layer, const hymba_block_weights *bw, int batch,
                                           int n_tokens, const void *x, void *y, hymba_kv_seq *kv,
                                           hymba_kv_cache *kv_cache, hymba_ssm_cache *ssm_cache,
                                           void *workspace, size_t workspace_bytes, hymba_stream_t stream);
HYMBA_API hymba_status hymba_block_decode_workspace(const hymba_layer *layer, int mlp_hidden, int batch,
                                                    int64_t max_pos, size_t *bytes);
/* The block for one new row per sequence: x_t, y_t [batch, d_model] dtype (distinct);
 * other arguments as for hymba_layer_decode_step. */
HYMBA_API hymba_status hymba_block_decode_step(hymba_layer *layer, const hymba_block_weights *bw, int batch,
                                               int64_t pos, const void *x_t, void *y_t,
                                               hymba_kv_cache *kv_cache, hymba_ssm_cache *ssm_cache,
                                               void *workspace, size_t workspace_bytes, hymba_stream_t stream);

/* ---- status and diagnostics -------------------------------------------- */

/* Synchronises `stream`, then reports a pending CUDA error or a device-side
 * error word (e.g. a bounded wait that timed out) and clears the word. */
HYMBA_API hymba_status hymba_stream_status(hymba_stream_t stream);
/* Bounded device waits.  Every wait of the tensor-core kernels on an mbarrier (a TMA
 * copy, an MMA, a pipeline stage) gives up after a limit in SM clock cycles, records a
 * timeout in the library's device error word, drains what its CTA has in flight, releases
 * its tensor memory and returns; hymba_stream_status() then reports HYMBA_ERR_TIMEOUT.
 * This sets the limit for launches issued from now on: `cycles` >= 1e5 (smaller values
 * are raised to 1e5); 0 restores the default, which is the HYMBA_WAIT_LIMIT environment
 * variable when set, else 1e9 cycles (about half a second).  *applied (optional) receives
 * the limit now in force.  Host only; not a hot call. */
HYMBA_API hymba_status hymba_set_wait_limit(int64_t cycles, int64_t *applied);

/* Diagnostic of the bounded-wait path: in the next `count` calls of hymba_layer_prefill
 * (bf16 path), the output projection's MMA warp waits for an arrival that never comes
 * instead of issuing its first MMA, so that kernel's waits run out: it records a timeout,
 * drains and returns (its output rows are then undefined), and hymba_stream_status()
 * reports HYMBA_ERR_TIMEOUT.  No fault and no unbounded wait is involved.  0 cancels. */
HYMBA_API hymba_status hymba_debug_stall_next_prefill(int count);

/* Reason for the last non-OK status returned on this thread ("" if none). */
HYMBA_API const char *hymba_last_error(void);
HYMBA_API const char *hymba_status_string(hymba_status s);
/* Library version, e.g. "hymba-b200 0.1 sm_100a". */
HYMBA_API const char *hymba_version(void);

/* The prefill attention mask exactly as an attention kernel applies it, for bit-exact
 * checks against the definition (Hymba §2.1 Eq. 1 under the A-shape mask of the authors'
 * OpenReview reply, or causal for a global layer, §2.2).
 *   path 0: the bf16 tensor-core kernel: a key is visible iff its 128-key tile is among
 *           the tiles the kernel streams for the query's pair of 128-row tiles, the
 *           tile's class is not "skipped", and (partially visible tile) its column is
 *           in the keep-mask the softmax applies.  The dump calls the kernel's own
 *           device functions for each of these decisions.
 *   path 1: the fp32 CUDA-core kernel: its per-pair predicate.
 * bits [L, ceil(L/32)] uint32 (device) row-major: bit j%32 of word j/32 of row i is 1 iff
 * key j is visible from query i.  tile_class (optional, device) [ceil(L/128)]^2 uint8:
 * 0 = skipped (no visible pair), 1 = fully visible, 2 = partially masked, as the tensor-
 * core kernel classifies 128x128 tiles.  INVALID_ARG for a bad shape or path. */
HYMBA_API hymba_status hymba_debug_mask_bitmap(int L, int n_meta, int window, int is_global, int path,
                                               uint32_t *bits, uint8_t *tile_class,
                                               hymba_stream_t stream);

/* The decode attention's key-slot mask for the query at X~ position `pos` (the predicate
 * both decode kernels apply to every slot of the K/V store; slot rule as for
 * hymba_kv_cache).  bits [ceil(capacity/32)] uint32 (device): bit s%32 of word s/32 is 1
 * iff slot s holds a position visible from pos.  capacity must cover the slots the query
 * reads (m + W, or pos + 1 for a global layer), else INVALID_ARG. */
HYMBA_API hymba_status hymba_debug_decode_mask(int64_t pos, int n_meta, int window, int is_global,
                                               int capacity, uint32_t *bits, hymba_stream_t stream);

/* 2^x of n floats (device buffers) by the FMA-pipe polynomial (degree 3 or 5) that the
 * prefill attention softmax uses for a share of its exponentials.  For checking the
 * stated bound: relative error <= 7.5e-5 (degree 3) or 2.4e-7 (degree 5) for
 * -125 <= x < 128 beyond fp32 rounding; x < -125 returns 2^-125. */
HYMBA_API hymba_status hymba_debug_exp2_poly(int degree, const float *x, float *y, int64_t n,
                                             hymba_stream_t stream);

/* ---- optional per-kernel timing ---------------------------------------- */

/* When enabled, every kernel launch issued by the compute calls (outside CUDA
 * graph capture) is bracketed by two CUDA events on its stream; the events come
 * from a pool created here, so enabling is not a hot call.  Disabled by default. */
HYMBA_API hymba_status hymba_profile_enable(int on);
typedef struct {
  char name[32];     /* pipeline step, e.g. "in_proj", "attention", "scan" */
  int calls;         /* times the step ran */
  int kernels;       /* kernels it launched in total */
  double total_ms;   /* sum of event-measured durations */
} hymba_profile_entry;
/* Synchronises the recorded events, accumulates them per step name and clears
 * the record.  Writes up to `max` entries, *n = number written. */
HYMBA_API hymba_status hymba_profile_collect(hymba_profile_entry *out, int max, int *n);

#ifdef __cplusplus
}
#endif
#endif /* HYMBA_H_ */
