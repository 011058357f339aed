/*
 * librswa -- Reference Sliding Window Attention (R-SWA) decode hot path for
 * NVIDIA B200 (sm_100a), behind a plain C ABI.
 *
 * Method source (cited by page title and section):
 *   "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" (gtnt.cn)
 *     §2.1 环形滑窗注意力 -- the KV cache keeps every prefill token at full
 *          attention plus a ring of the W most recently generated tokens.
 *          Generated tokens are appended until the cache holds prefill_len + W
 *          entries; from then on each new token overwrites slot
 *          prefill_len + ring_pos and ring_pos advances by one modulo W.  The
 *          token then attends to the whole cache, whose size stays at
 *          prefill_len + W however long the output runs.  W is
 *          sliding_window_size = 128 in the model's config.
 *     §2.3 反循环采样 -- inside a sliding window of the generated history,
 *          every token that would repeat an n-gram of size ngram_size gets
 *          score -inf (defaults no_repeat_ngram_size 35, ngram_window 128).
 *     §三  -- the transformers path materialises the full prefill score
 *          matrix; a flash-style ring implementation is named as open work.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named "device" are CUDA device pointers on the current device;
 *    pointers named "host" are ordinary host memory.  `stream` is a
 *    cudaStream_t (NULL = legacy default stream).  All device work is enqueued
 *    asynchronously on `stream`; only rswa_state_create, rswa_get_ring and
 *    rswa_check_device_error synchronise.
 *  - OWNERSHIP: the caller owns ALL device memory (inputs, outputs, K/V
 *    caches, workspace).  The library never allocates or frees device memory;
 *    it keeps raw pointers inside the opaque host-side state.
 *  - ERRORS: argument problems found on the host return RSWA_EINVAL before
 *    anything is enqueued.  A failed launch returns RSWA_ECUDA.  Problems the
 *    kernels find (a token id outside the vocabulary, a wait that ran out)
 *    are recorded in a device error word and reported by
 *    rswa_check_device_error (or, for rswa_ngram_mask, in the caller's
 *    `device_error` word).  Nothing traps, aborts or waits without a bound.
 *  - Element types: RSWA_BF16 (bfloat16, round-to-nearest-even outputs with
 *    fp32 accumulation) or RSWA_F32.  head_dim is 64 or 128.
 *  - Heads: multi-head attention, num_kv_heads == num_heads.  Positions: by
 *    default keys are stored and used exactly as given (the caller applies
 *    any position encoding); rswa_state_set_rope moves the rotary embedding
 *    into the library, applied when keys enter the cache.
 *
 * Layouts
 * -------
 *  Token-major activations: q, k, v, out of the prefill are packed varlen
 *  [sum_b P_b][H][d]; decode q, k_new, v_new, out are [B][H][d]; rows are
 *  contiguous, d fastest.
 *
 *  K/V cache of one layer (one buffer for K, one for V, rswa_cache_bytes()
 *  each): sequence-major, then head-major, then slot:
 *      element offset of (b, h, slot, e) =
 *          (H * S_b + h * (P_b + W) + slot) * d + e,
 *      S_b = sum_{b' < b} (P_b' + W),   0 <= slot < P_b + W.
 *  Slots [0, P_b) hold the prefill; slots [P_b, P_b + W) hold the ring.
 *  rswa_cache_offset() returns this offset.  Every (b, h) ring of the cache
 *  is contiguous, so it is streamed with 16-byte-aligned bulk copies.
 */
#ifndef RSWA_H
#define RSWA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RSWA_ABI_VERSION 1

typedef enum rswa_status {
  RSWA_OK = 0,
  RSWA_EINVAL = 1,   /* bad argument (null pointer, size, dtype, range)      */
  RSWA_ENOMEM = 2,   /* caller-provided workspace smaller than required      */
  RSWA_ECUDA = 3,    /* a CUDA runtime call or kernel launch failed          */
  RSWA_ESTATE = 4,   /* call out of order (decode before prefill, ...)       */
  RSWA_ETIMEOUT = 5, /* a kernel's bounded wait ran out (device error word)  */
  RSWA_EDEVICE = 6   /* a kernel rejected its data (device error word)       */
} rswa_status;

typedef enum rswa_dtype { RSWA_F32 = 0, RSWA_BF16 = 1 } rswa_dtype;

/* Model/batch shape shared by every layer. */
typedef struct rswa_config {
  int32_t batch;      /* B >= 1 sequences                                    */
  int32_t num_layers; /* >= 1; each layer has its own K and V cache buffer   */
  int32_t num_heads;  /* H >= 1                                              */
  int32_t head_dim;   /* d in {64, 128}                                      */
  int32_t window;     /* W >= 1 ring entries (the pages use 128)             */
  int32_t dtype;      /* rswa_dtype of q/k/v/out and of the caches           */
  float scale;        /* softmax scale; 0 selects 1/sqrt(head_dim)           */
} rswa_config;

/* Opaque host-side state: shape, raw device pointers, work decomposition. */
typedef struct rswa_state rswa_state;

/* Bytes of ONE cache buffer (K or V) of ONE layer:
 *   H * d * elem_size * sum_b (P_b + W).
 * prefill_len: host [B], each >= 0.  Returns 0 if the arguments are invalid. */
size_t rswa_cache_bytes(const rswa_config *cfg, const int64_t *prefill_len);

/* Bytes of device workspace rswa_state_create needs (error word, per-sequence
 * counters, the split-K work list, split-K partials).  Depends on the device's
 * SM count, so call it with the target device current.  0 if invalid. */
size_t rswa_workspace_bytes(const rswa_config *cfg, const int64_t *prefill_len);

/* Build the state for one batch.
 *  prefill_len : host [B], P_b >= 0, P_b + W < 2^31.
 *  n_generated : host [B] or NULL.  NULL: a fresh batch; every layer must be
 *                filled by rswa_prefill before its first rswa_decode_step.
 *                Non-NULL: resume a batch whose caches the caller has already
 *                filled (prefill slots and the first min(n, W) ring slots, in
 *                the layout above) after n_generated[b] tokens; decode may
 *                start at once on every layer.
 *  k_cache, v_cache : host arrays of num_layers device pointers, each to
 *                rswa_cache_bytes() bytes, 16-byte aligned.
 *  workspace   : device pointer to workspace_size >= rswa_workspace_bytes()
 *                bytes, 256-byte aligned; owned by the caller, used by the
 *                state until rswa_state_destroy.
 *  stream      : the tables are uploaded on it; the call synchronises it.
 *  out         : receives the new state.
 * Returns RSWA_EINVAL, RSWA_ENOMEM (workspace too small) or RSWA_ECUDA. */
rswa_status rswa_state_create(const rswa_config *cfg, const int64_t *prefill_len,
                              const int64_t *n_generated, void *const *k_cache,
                              void *const *v_cache, void *workspace, size_t workspace_size,
                              void *stream, rswa_state **out);

/* ------------------------------------------------------------------------
 * Token pool and continuous batching [§三: serving with a page size of one
 * token].  Each request owns P_b + W cache slots for its whole life, so a
 * serving process keeps one K/V pool per layer and gives each joining request
 * one contiguous slot range, freed when the request leaves.  Requests join
 * and leave between decode steps: the caller builds a state over the requests
 * running now (rswa_state_create_pooled, with each request's slot base and its
 * current n_generated from rswa_get_ring of the previous state) and destroys
 * the old one; a joining request's prompt is filled by rswa_prefill of a
 * state over the joining requests alone, pointing at the same pool.
 * ------------------------------------------------------------------------ */
typedef struct rswa_pool rswa_pool;

/* Host-side allocator of slot ranges in a pool of `capacity` slots
 * (1 <= capacity < 2^40).  Allocation is first fit: the lowest base with
 * enough free slots after it.  Freed ranges merge with free neighbours.
 * Thread-safe.  No device memory is involved. */
rswa_status rswa_pool_create(int64_t capacity, rswa_pool **out);
rswa_status rswa_pool_destroy(rswa_pool *pool);
/* `slots` >= 1 contiguous slots; *base receives the first.  RSWA_ENOMEM when
 * no free range is long enough (the pool is unchanged). */
rswa_status rswa_pool_alloc(rswa_pool *pool, int64_t slots, int64_t *base);
/* Free the range that rswa_pool_alloc returned at `base`; RSWA_EINVAL if
 * `base` is not the start of an allocated range. */
rswa_status rswa_pool_free(rswa_pool *pool, int64_t base);
/* Any pointer may be NULL: free slots, longest free range, number of free
 * ranges, number of allocated ranges. */
rswa_status rswa_pool_stats(const rswa_pool *pool, int64_t *free_slots, int64_t *largest_free,
                            int32_t *n_free_ranges, int32_t *n_allocated);
/* Capacity in slots, or -1 for NULL. */
int64_t rswa_pool_capacity(const rswa_pool *pool);

/* Bytes of ONE pool cache buffer (K or V) of ONE layer holding `pool_slots`
 * slots: pool_slots * H * d * elem_size.  0 if invalid.  The batch field of
 * cfg is ignored. */
size_t rswa_pool_cache_bytes(const rswa_config *cfg, int64_t pool_slots);

/* As rswa_state_create, for requests placed anywhere in a pool:
 *  slot_base  : host [B] or NULL.  Request b's cache is slots
 *               [slot_base[b], slot_base[b] + P_b + W) of the pool, laid out
 *               head-major like the packed layout with S_b = slot_base[b]:
 *                 element offset of (b, h, slot, e) =
 *                     (H * slot_base[b] + h * (P_b + W) + slot) * d + e.
 *               NULL: packed back to back (pool_slots is then ignored).
 *  pool_slots : slots each cache buffer holds (rswa_pool_cache_bytes).
 * Returns RSWA_EINVAL if a range leaves [0, pool_slots) or two requests'
 * ranges overlap.  The workspace size is rswa_workspace_bytes(cfg,
 * prefill_len), as for a packed batch. */
rswa_status rswa_state_create_pooled(const rswa_config *cfg, const int64_t *prefill_len,
                                     const int64_t *n_generated, const int64_t *slot_base,
                                     int64_t pool_slots, void *const *k_cache,
                                     void *const *v_cache, void *workspace, size_t workspace_size,
                                     void *stream, rswa_state **out);

/* ------------------------------------------------------------------------
 * Rotary position embedding at cache-write time.  The pages fix the cache
 * (the prompt plus a ring of the W latest generated tokens; the model has
 * max_position_embeddings = 32768, §2.1) but not the position a generated
 * token takes once the ring has wrapped; the caller chooses:
 *   RSWA_ROPE_ABSOLUTE : generated token t (0-based) of request b sits at
 *                        position P_b + t -- the usual decoding positions;
 *   RSWA_ROPE_SLOT     : it sits at the cache slot it is written to,
 *                        P_b + (t mod W), so positions stay below P_b + W.
 * Prompt token i is at position i under both.  The rotation is rotate-half
 * (Llama family): for i < d/2 the pair (x_i, x_{i+d/2}) turns by the angle
 * pos * theta^(-2i/d) (angles reduced in double precision, the rotation in
 * float).  With RoPE on:
 *  - rswa_prefill rotates k into the cache and q into `out` (used as
 *    scratch: each query row is read there before its output overwrites it),
 *    and attends with the rotated q and k; v is not rotated;
 *  - rswa_decode_step rotates k_new before it enters the ring slot and q
 *    before it is used, both at the token's position;
 *  - the cache holds rotated keys (a resumed state's caller must have
 *    rotated the keys it filled in the same way).
 * ------------------------------------------------------------------------ */
typedef enum rswa_rope_policy {
  RSWA_ROPE_NONE = 0,
  RSWA_ROPE_ABSOLUTE = 1,
  RSWA_ROPE_SLOT = 2
} rswa_rope_policy;

/* Turn RoPE on (or off with RSWA_ROPE_NONE) for this state.  theta > 0 (the
 * Llama default is 10000).  Call it before the state's first rswa_prefill or
 * rswa_decode_step; it enqueues a small kernel on `stream`.  Returns
 * RSWA_EINVAL for a bad policy or theta. */
rswa_status rswa_state_set_rope(rswa_state *state, int32_t policy, float theta, void *stream);

/* ------------------------------------------------------------------------
 * Standard sliding-window attention, the contrast the pages draw [§2.1: a
 * standard sliding window would cut the prefill K/V as well, which for OCR
 * loses image tokens; R-SWA keeps the whole prompt].  In this mode every
 * token -- prompt and generated -- attends to the last W positions only,
 * itself included: prompt query i to keys max(0, i - W + 1) .. i, and the
 * t-th generated token (position P_b + t) to positions P_b + t - W + 1 ..
 * P_b + t, i.e. the last W - 1 - t prompt tokens while t < W - 1 plus the
 * ring.  The cache layout, the ring writes and rswa_advance are unchanged:
 * the mode changes what is attended, not what is stored.  The prefill visits
 * only the key tiles of each query tile's window; decode gives each ring a
 * cluster of ceil(W / 64) CTAs.
 * ------------------------------------------------------------------------ */
typedef enum rswa_attention_mode {
  RSWA_ATTN_RING = 0,          /* R-SWA (default) */
  RSWA_ATTN_STANDARD_SWA = 1   /* the window also cuts the prompt */
} rswa_attention_mode;

/* Takes effect for the calls enqueued after it.  Switching mode re-uploads
 * the prefill work list with a synchronous copy (call it before enqueuing
 * work, not between calls in flight).  RSWA_EINVAL for an unknown mode. */
rswa_status rswa_state_set_attention(rswa_state *state, int32_t mode);

/* ------------------------------------------------------------------------
 * Key-range split of one long sequence's cache over G devices.  Softmax
 * attention over a key set is the log-sum-exp merge of its value over the
 * parts of any partition of the set, so G shares of the cache can each
 * produce a partial (m, l, o) and one merge gives the decode output.  A
 * process per device holds its share as an ordinary state (its slice of the
 * prompt as prefill_len; the last share also holds the ring), calls
 * rswa_decode_step_partial, exchanges the partials (G x B x H x (d + 2)
 * floats, e.g. an all-gather over NCCL), and calls rswa_combine_partials.
 * The ring write of a step is done by the share whose range holds the slot.
 * RoPE in the library follows each state's own positions, so a split
 * sequence rotates its keys and queries before the calls (or all shares but
 * the first would rotate at shifted positions).
 * ------------------------------------------------------------------------ */

/* rswa_decode_step restricted to cache slots [key_lo, key_hi) of every ring
 * (intersected with the entries held), writing the unnormalised partial:
 *  part_ml : device float [B][H][2]: m (the running max, in log2 units:
 *            max of scale*log2(e)*q.k) and l = sum 2^(s - m); an empty range
 *            gives m = -inf, l = 0;
 *  part_o  : device float [B][H][d]: sum 2^(s - m) v.
 * The step's ring write happens only if its slot lies in the range.  16-byte
 * aligned pointers.  RSWA_EINVAL for a bad range or pointer, RSWA_ESTATE as
 * rswa_decode_step. */
rswa_status rswa_decode_step_partial(rswa_state *state, int32_t layer, const void *q,
                                     const void *k_new, const void *v_new, int64_t key_lo,
                                     int64_t key_hi, float *part_ml, float *part_o,
                                     void *stream);

/* Merge `shares` partials per ring: part_ml device float [shares][rings][2],
 * part_o device float [shares][rings][head_dim] -> out [rings][head_dim] of
 * `dtype` (RSWA_F32 or RSWA_BF16): out = sum_g 2^(m_g - M) o_g /
 * sum_g 2^(m_g - M) l_g with M = max_g m_g.  rings = B * H. */
rswa_status rswa_combine_partials(const float *part_ml, const float *part_o, int32_t shares,
                                  int64_t rings, int32_t head_dim, int32_t dtype, void *out,
                                  void *stream);

/* Free the host-side state.  Device memory stays the caller's. */
rswa_status rswa_state_destroy(rswa_state *state);

/* Element offset of (b, h, slot, 0) inside one layer's cache buffer, or -1. */
int64_t rswa_cache_offset(const rswa_state *state, int32_t b, int32_t h, int64_t slot);

/* Prefill of one layer [§2.1: the prefill segment keeps full attention].
 *  q, k, v : device [sum_b P_b][H][d] (packed varlen, sequence b's tokens at
 *            rows sum_{b'<b} P_b' ...), dtype of the config.
 *  out     : device [sum_b P_b][H][d]: causal softmax attention of each token
 *            over tokens 0..i of its own sequence (no window).
 * Also stores k, v into cache slots [0, P_b) of this layer; the ring
 * counters are not touched.  All pointers 16-byte aligned.  Returns
 * RSWA_EINVAL for a bad layer or pointer. */
rswa_status rswa_prefill(rswa_state *state, int32_t layer, const void *q, const void *k,
                         const void *v, void *out, void *stream);

/* One decode step of one layer [§2.1 steady-state/warm-up phases].
 *  q, k_new, v_new, out : device [B][H][d].
 * For each sequence b with t_b tokens generated so far (t_b is device
 * resident, advanced by rswa_advance):
 *   slot  = P_b + (t_b mod W)     -- the warm-up append and the steady-state
 *                                    ring overwrite are the same formula;
 *   cache[slot] <- (k_new, v_new);
 *   out   = softmax attention of q over slots [0, P_b + min(t_b + 1, W)).
 * The write, the attention and the split-K combine are one kernel.  Safe to
 * capture in a CUDA graph (no host-side state changes per step).
 * The kernel uses programmatic dependent launch: it may start while the
 * previous kernel in the stream is still running if that kernel lets its
 * dependents start early (griddepcontrol.launch_dependents), and it then
 * reads prompt rows (slots < P_b) of this layer's cache before waiting for
 * that kernel.  A kernel that writes prompt rows must therefore not release
 * its dependents early; everything else is read after the wait.  (Before the
 * wait it also asks L2 for the lines of q, k_new, v_new and t_b: a prefetch
 * returns nothing, so rows an earlier kernel is still writing are read fresh
 * after the wait.)
 * RSWA_ESTATE if the layer was never prefilled. */
rswa_status rswa_decode_step(rswa_state *state, int32_t layer, const void *q, const void *k_new,
                             const void *v_new, void *out, void *stream);

/* t_b += 1 for every sequence, on the device: once per generated token, after
 * the token's last layer.  Capturable in a CUDA graph. */
rswa_status rswa_advance(rswa_state *state, void *stream);

/* Restore every t_b to its value at rswa_state_create (0, or n_generated),
 * on the device; capturable.  Starts the batch's generation over without
 * rebuilding the state (the caches are not touched). */
rswa_status rswa_reset_ring(rswa_state *state, void *stream);

/* Windowed no-repeat n-gram ban [§2.3].
 *  logits     : device fp32 [rows][ld], ld >= vocab; modified in place.
 *  history    : device int32 [rows][hist_ld], hist_ld >= window; row r holds
 *               its last h_r generated tokens, oldest first, in [0, h_r).
 *  hist_len   : device int32 [rows] (h_r, 0 <= h_r <= window) or NULL (all
 *               rows hold `window` tokens).
 *  n          : n-gram size >= 1 (the pages use 35); window >= 0 (128).
 *  device_error : device int32 or NULL; on bad row data the kernel ORs
 *               RSWA_DEVERR_BAD_TOKEN / RSWA_DEVERR_BAD_LENGTH into it.
 * For each row with h_r >= n: the next token x would form the n-gram
 * (hist[h_r-n+1 .. h_r-1], x); every start i in [0, h_r - n] whose (n-1)-gram
 * hist[i .. i+n-2] equals that prefix sets logits[r][hist[i+n-1]] = -inf.
 * Nothing else is written, bit for bit.  A row with h_r outside [0, window]
 * or a token outside [0, vocab) in [0, h_r) is left untouched.  Rows with
 * h_r < n, and window < n, ban nothing. */
rswa_status rswa_ngram_mask(float *logits, int64_t ld, const int32_t *history, int64_t hist_ld,
                            const int32_t *hist_len, int32_t rows, int32_t vocab, int32_t n,
                            int32_t window, int32_t *device_error, void *stream);

/* Fused n-gram ban + top-k selection, the step after the ban [§2.3: the
 * banned tokens score -inf and the next token is chosen from the masked
 * scores; greedy decoding at k = 1].
 * For each row r < rows, with the banned set of rswa_ngram_mask (same
 * history, hist_len, n, window and error rules), the masked row is
 * x_j = -inf for banned j, logits[r, j] otherwise (NaN ranks as -inf).
 * Columns are ordered by x_j descending, the lower column first among equal
 * values; the first k of that order are written:
 *  top_idx : device int32 [rows][k] (required);
 *  top_val : device float [rows][k] or NULL -- x of those columns.
 *  token   : device int32 [rows] or NULL -- the chosen token: with uniform
 *            NULL, top_idx[r][0] (greedy); otherwise the inverse CDF at
 *            uniform[r] of p_i proportional to exp((x_i - x_0) / temperature)
 *            over the k columns: the first i whose running sum of p exceeds
 *            uniform[r] * sum(p) (columns with x = -inf have p = 0).
 *  uniform : device float [rows] in [0, 1), or NULL; temperature > 0 when set.
 *  mask_in_place : nonzero also stores -inf into logits at the banned
 *            columns, as rswa_ngram_mask does; zero leaves logits untouched.
 * Limits: 1 <= k <= RSWA_TOPK_MAX and k <= vocab; vocab <= RSWA_TOPK_MAX_VOCAB;
 * window <= 8192 (the history is staged in shared memory);
 * ld >= vocab and ld a multiple of 4; logits 16-byte aligned (logits is
 * read as float4 up to column ceil(vocab / 4) * 4 - 1 of each row).  A row
 * whose history is invalid gets top_idx -1, top_val NaN and token -1, and the
 * error bit in device_error.  Each row is read from HBM once. */
#define RSWA_TOPK_MAX 64
#define RSWA_TOPK_MAX_VOCAB 262144
rswa_status rswa_ngram_topk(float *logits, int64_t ld, const int32_t *history, int64_t hist_ld,
                            const int32_t *hist_len, int32_t rows, int32_t vocab, int32_t n,
                            int32_t window, int32_t k, int32_t mask_in_place,
                            const float *uniform, float temperature, int32_t *top_idx,
                            float *top_val, int32_t *token, int32_t *device_error, void *stream);

/* Synchronises `stream`, then copies the ring counters to the host:
 *  n_generated : host [B] or NULL -- t_b;
 *  ring_pos    : host [B] or NULL -- the pages' ring_pos: 0 during warm-up,
 *                t_b mod W once the cache is full (next slot is P_b+ring_pos);
 *  cache_len   : host [B] or NULL -- entries held, P_b + min(t_b, W). */
rswa_status rswa_get_ring(const rswa_state *state, int64_t *n_generated, int32_t *ring_pos,
                          int64_t *cache_len, void *stream);

/* Synchronises `stream` and reads the state's device error word:
 * RSWA_OK, RSWA_ETIMEOUT or RSWA_EDEVICE.  Clears the word. */
rswa_status rswa_check_device_error(rswa_state *state, void *stream);

/* The launch shape rswa_decode_step uses for this state (host only, no
 * synchronisation):
 *  grid         : CTAs per decode launch;
 *  cluster_size : 0 when the flattened key rows of all rings are split into
 *                 `grid` equal ranges whose partials are merged through the
 *                 workspace; C >= 2 when each (b, h) ring has a cluster of C
 *                 CTAs that merge through distributed shared memory (chosen
 *                 when all rings' clusters are resident at once).
 * Either pointer may be NULL.  The environment variable RSWA_DECODE_SPLIT
 * (`streamk` or `cluster`), read by rswa_state_create, overrides the choice
 * where the cluster form fits. */
rswa_status rswa_decode_launch_shape(const rswa_state *state, int32_t *grid,
                                     int32_t *cluster_size);

/* Static description of a status code. */
const char *rswa_status_string(rswa_status status);

/* Description of the CUDA error behind the calling thread's most recent
 * RSWA_ECUDA ("no error" if there was none).  Static storage. */
const char *rswa_last_cuda_error(void);

/* ---- Allocation-free decode step --------------------------------------
 * This call has no counterpart in the method itself; it exists for callers that
 * cannot hand the library a workspace.  A plugin hosted by another runtime
 * or inference server gets its input and output tensors but may not allocate
 * device memory itself (the host application's allocator owns the pool, so a
 * private cudaMalloc can fail or fragment it), and a latency-bound serving
 * loop keeps cudaMalloc/cudaFree off its hot path because both can
 * synchronise the device.
 *
 * Same computation as rswa_decode_step for ONE layer, without a state: the
 * caller passes the ring position explicitly and advances it itself.  It is
 * always the ring attention of the method, with keys and queries used as
 * given: the RoPE and attention-mode settings of rswa_state_set_rope and
 * rswa_state_set_attention belong to a state and do not apply here.
 *  cfg           : as for rswa_state_create (num_layers is ignored).
 *  prefill_len   : host [B], P_b.
 *  n_generated   : host [B], t_b = tokens generated before this step; the
 *                  step writes slot P_b + (t_b mod W) and attends over
 *                  slots [0, P_b + min(t_b + 1, W)).
 *  k_cache, v_cache : device, this layer's caches in the layout above.
 *  q, k_new, v_new, out : device [B][H][d].  All device pointers 16-byte aligned.
 *  device_error  : device int32 or NULL; kernel error bits are ORed into it
 *                  (NULL: they go to a word inside the scratch, cleared by
 *                  each call, and are not reported).
 * Scratch: a file-scope device array of RSWA_NOALLOC_SCRATCH_BYTES bytes on
 * every device that loads the library, held until the process exits.  The
 * call allocates nothing (no cudaMalloc/cudaFree).  Its first call on a
 * device looks up the array's device address (cudaGetSymbolAddress); make
 * that first call before any stream capture.  At every call the work tables
 * are written into the array by small kernels enqueued on `stream` that carry
 * the bytes in their launch parameters, so no host memory is referenced once
 * the call has returned.  Every call on a device shares the one array and it
 * keeps the last call's contents, so calls whose work overlaps on the GPU
 * (different streams, no ordering) race and corrupt each other; order them
 * on one stream.
 * Returns RSWA_EINVAL for bad arguments and RSWA_ENOMEM when the batch needs
 * more scratch than the array holds.  What counts is the decode step's part of
 * a workspace: error word, ring counters, P_b, slot bases, the split-K work
 * tables and the partials.  The keys of all rings are cut into one range per
 * decode CTA (3 per SM), so there are at most (CTAs + B*H) pieces, each
 * taking 32 bytes of table and 8 + 4d bytes of partials: about 0.6 MiB for
 * 64 requests of 10 heads at d = 128 on a 148-SM part, whatever the prompt
 * lengths; about 7,000 (b, h) rings of d = 128 fit. */
#define RSWA_NOALLOC_SCRATCH_BYTES (4u << 20)
rswa_status rswa_decode_step_noalloc(const rswa_config *cfg, const int64_t *prefill_len,
                                     const int64_t *n_generated, void *k_cache, void *v_cache,
                                     const void *q, const void *k_new, const void *v_new,
                                     void *out, int32_t *device_error, void *stream);

/* ---- Fault injection (tests only) ---------------------------------------
 * RSWA_FAULT_DROP_DECODE_COPIES: subsequent decode kernels of this state
 * issue none of their cache copies, so every bounded wait in them runs out
 * (about 1 s): the kernel records RSWA_DEVERR_TIMEOUT, finishes, and
 * rswa_check_device_error returns RSWA_ETIMEOUT; outputs of those steps are
 * garbage, the cache is untouched apart from the ring write.
 * RSWA_FAULT_DROP_PREFILL_LOADS: subsequent tensor-core prefills (bf16,
 * d = 128) of this state issue none of their tile loads: every bounded wait
 * runs out, the kernel records RSWA_DEVERR_TIMEOUT, frees its tensor memory
 * and returns; the outputs and the cache's prompt slots of those calls are not
 * written.  flags = 0 restores normal operation.  Enqueued on `stream`
 * (pageable copy). */
#define RSWA_FAULT_DROP_DECODE_COPIES 1
#define RSWA_FAULT_DROP_PREFILL_LOADS 2
rswa_status rswa_debug_inject_fault(rswa_state *state, int32_t flags, void *stream);

/* ---- Prefill work plan (tests only) ---------------------------------------
 * The blocks the tensor-core prefill (bf16, d = 128) would launch for this
 * batch on a part with `num_sms` SMs, in launch order: 4 int32 per block,
 * (request b, head h, first query tile, query tiles 1 or 2), into `out`
 * (host, room for `capacity` blocks).  Host only: no device is touched.
 * Returns the number of blocks (those past `capacity` are not written), or
 * -1 for a bad config or arguments. */
int64_t rswa_debug_prefill_plan(const rswa_config *cfg, const int64_t *prefill_len,
                                int32_t num_sms, int32_t *out, int64_t capacity);

/* Bits of a device error word. */
#define RSWA_DEVERR_TIMEOUT 1
#define RSWA_DEVERR_BAD_TOKEN 2
#define RSWA_DEVERR_BAD_LENGTH 4

#ifdef __cplusplus
}
#endif

#endif /* RSWA_H */
