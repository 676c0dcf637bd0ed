/*
 * h2okv.h -- C ABI of the B200 (sm_100a) chunked KV-cache attention library
 * with H2O score-sum, eviction and 8/4-bit cache quantization.
 *
 * The operations follow "Learning how to Forget: Fine-tuning for Long-Context
 * Sparse Attention" (the KeysAndValues paper):
 *   - §3.1: one layer's cache is the buffers keys, values (B, H_k, N_C, d_h) and
 *     token_pos (B, H_k, N_C); it fills left to right, then a per-(b, h) policy
 *     picks the slots that each chunk of S new tokens overwrites;
 *   - §A.1: SDPA for tokens P..P+S-1 masks slot j of head (b, h) when
 *     P + i < token_pos[b, h, j]; the chunk's keys/values are written first;
 *   - §A.7: SDPA is softmax(mask(d_h^-1/2 Q K^T)) V and also returns the
 *     attention weights summed over the query axis, shape (B, H_q, N_k);
 *   - §3.1.1: the H2O score of an entry is the running sum of those weights
 *     while it is cached; the lowest score is evicted;
 *   - §2 / §A.10: cache buffers may be quantized to 8 or 4 bits.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers unless stated otherwise; the
 *     caller allocates and owns them (and the stream).  The handle owns only
 *     host-side metadata.
 *   - Tensors are dense, row-major, innermost dimension last, no padding.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work; they never synchronize the device.
 *   - Return value: H2OKV_OK (0) or a negative error code.  Arguments are
 *     validated on the host before anything is enqueued; on error nothing is
 *     enqueued and h2okv_last_error() returns a message (thread-local).
 *     Kernels never trap.
 *   - GQA: query head h belongs to KV head (group) h / q_g, q_g = H_q / H_k.
 *   - Token positions are int32; a slot holding no token stores INT32_MAX.
 */
#ifndef H2OKV_H
#define H2OKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define H2OKV_API __attribute__((visibility("default")))
#else
#define H2OKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes ------------------------------------------------------- */
#define H2OKV_OK 0
#define H2OKV_ERR_INVALID_ARG (-1) /* bad pointer, size, shape or dtype combination */
#define H2OKV_ERR_UNSUPPORTED (-2) /* valid request this build does not implement   */
#define H2OKV_ERR_CUDA (-3)        /* a CUDA runtime/driver call or launch failed    */
#define H2OKV_ERR_TIMEOUT (-4)     /* a bounded device-side wait gave up             */

/* ---- element types ----------------------------------------------------- */
#define H2OKV_F32 0  /* float32                                              */
#define H2OKV_BF16 1 /* bfloat16                                             */
#define H2OKV_I8 2   /* int8 codes + one fp16 scale per (b, h_k, slot) row    */
#define H2OKV_I4 3   /* int4 codes, two per byte (even element in the low
                        nibble, two's complement) + one fp16 scale per row    */

/* empty-slot token position */
#define H2OKV_EMPTY_POS INT32_MAX

typedef struct h2okv_cache h2okv_cache; /* opaque handle */

/* Shape and types of one layer's cache (§3.1). */
typedef struct {
  int32_t batch;      /* B >= 1                                               */
  int32_t n_q_heads;  /* H_q, a multiple of n_kv_heads                        */
  int32_t n_kv_heads; /* H_k >= 1                                             */
  int32_t head_dim;   /* d_h: a multiple of 8, 8..256                         */
  int32_t capacity;   /* N_C: 1..65536 slots                                  */
  int32_t max_chunk;  /* largest S any call on this cache will pass (sizes the
                         workspace)                                           */
  int32_t q_dtype;    /* H2OKV_F32 or H2OKV_BF16: dtype of q, y and of new
                         keys/values                                          */
  int32_t kv_dtype;   /* storage dtype of keys/values: F32 (needs q_dtype F32),
                         BF16, I8 or I4 (need q_dtype BF16)                   */
} h2okv_cache_desc;

/* Device buffers of one cache; sizes from kv_cache_query_sizes(). */
typedef struct {
  void *keys;         /* [B, H_k, N_C, d_h] in kv_dtype (I4: d_h/2 bytes/row) */
  void *values;       /* same layout as keys                                  */
  void *k_scales;     /* [B, H_k, N_C] fp16 for I8/I4, else NULL              */
  void *v_scales;     /* [B, H_k, N_C] fp16 for I8/I4, else NULL              */
  int32_t *token_pos; /* [B, H_k, N_C] int32                                  */
  float *scores;      /* [B, H_k, N_C] float32 cumulative H2O scores          */
  void *workspace;    /* scratch; contents need no initialisation; 256-byte
                         aligned; must not be shared by two caches whose calls
                         can run concurrently                                 */
} h2okv_cache_buffers;

enum {
  H2OKV_BUF_KEYS = 0,
  H2OKV_BUF_VALUES,
  H2OKV_BUF_K_SCALES,
  H2OKV_BUF_V_SCALES,
  H2OKV_BUF_TOKEN_POS,
  H2OKV_BUF_SCORES,
  H2OKV_BUF_WORKSPACE,
  H2OKV_NUM_BUFS
};

/* Byte size of each buffer of a cache with this description, indexed by
 * H2OKV_BUF_*; 0 for a buffer the dtype does not use.  Host only. */
H2OKV_API int kv_cache_query_sizes(const h2okv_cache_desc *desc, size_t sizes[H2OKV_NUM_BUFS]);

/* Create a handle over caller-owned buffers and enqueue their initialisation
 * on `stream`: token_pos = INT32_MAX (empty), scores = 0, keys/values/scales
 * zero-filled (the attention kernels read every slot and mask empty ones
 * arithmetically, so every slot must hold finite values; a caller that writes
 * the buffers directly must keep them finite).  The cache then holds no token
 * (fill level 0).  Writes the handle to *out. */
H2OKV_API int kv_cache_create(const h2okv_cache_desc *desc, const h2okv_cache_buffers *bufs,
                    void *stream, h2okv_cache **out);

/* Return the cache to the empty state (token_pos and scores as after create;
 * the rows keep their previous, finite contents). */
H2OKV_API int kv_cache_reset(h2okv_cache *cache, void *stream);

/* Free the handle (not the caller's buffers).  NULL is accepted. */
H2OKV_API int kv_cache_destroy(h2okv_cache *cache);

/* Fill level bookkeeping: the number of occupied slots.  The library keeps it
 * on the host; set it after writing a cache state into the buffers directly
 * (occupied slots must then be exactly those with token_pos != INT32_MAX).
 * While the eviction policy fills the cache left to right the attention scans
 * only the slots filled so far; kv_cache_set_fill and h2o_insert_at make it
 * scan every slot from then on (until kv_cache_reset). */
H2OKV_API int kv_cache_get_fill(const h2okv_cache *cache, int32_t *n_filled);
H2OKV_API int kv_cache_set_fill(h2okv_cache *cache, int32_t n_filled);

/* Device status of a cache: the tensor-core kernels bound every wait on
 * another warp or on a copy; when a wait exceeds the cache's limit the kernel
 * stops early, drains its own copies and matrix operations, frees its tensor
 * memory and records H2OKV_ERR_TIMEOUT here (outputs of that call are then
 * undefined).  This call synchronizes `stream`, returns the recorded status
 * (0 = ok) in *status and clears it. */
H2OKV_API int kv_cache_device_status(h2okv_cache *cache, int32_t *status, void *stream);

/* Limit of each bounded device-side wait, in nanoseconds (default 2 s).  A
 * limit of 0 makes the first wait that does not complete at once give up:
 * use it only to exercise the timeout path. */
H2OKV_API int kv_cache_set_wait_timeout(h2okv_cache *cache, uint64_t timeout_ns);

/* Quantize n_rows rows of head_dim bf16 values (the 8/4-bit cache format, §2 /
 * §A.10; the paper gives only the bit width, the scheme is):
 *   scale = fp16_rn(min(absmax / qmax, 65504)), qmax = 127 (I8) or 7 (I4);
 *   code  = clamp(rint(x / scale), -qmax, qmax); scale 0 gives codes 0.
 * All divisions are IEEE float32.  x_bf16: [n_rows, head_dim] bf16 (device).
 * codes_out: [n_rows, head_dim] int8 (I8) or [n_rows, head_dim/2] bytes (I4).
 * scales_out: [n_rows] fp16.  kv_dtype: H2OKV_I8 or H2OKV_I4. */
H2OKV_API int kv_cache_quantize(int32_t kv_dtype, const void *x_bf16, int64_t n_rows, int32_t head_dim,
                      void *codes_out, void *scales_out, void *stream);

/* H2O score update, slot choice and overwrite for one chunk (§3.1, §3.1.1,
 * §A.5.3 keys' = scatter(keys, index, key_new)), per (b, h_k):
 *   1. if w_prev != NULL: scores = float32(scores + w_prev)
 *      (w_prev: [B, H_k, N_C] float32, normally the previous chunk's w_out);
 *   2. choose S slots: empty slots first (lowest index first), then the
 *      occupied slots with the smallest (key, slot index) pairs -- lowest key,
 *      ties to the lowest index; the key is the score, or the variant set by
 *      kv_cache_set_score_mode;
 *   3. chunk token k (position P + k) goes to the k-th smallest chosen slot:
 *      keys/values rows <- k_new/v_new row k (quantized for I8/I4),
 *      token_pos = P + k, scores = 0;
 *   4. if slots_out != NULL: slots_out[b, h_k, k] = that slot (int32).
 * k_new, v_new: [B, H_k, S, d_h] in q_dtype (bf16 for BF16/I8/I4 caches).
 * S = 0 performs step 1 only (k_new/v_new/slots_out may be NULL): use it to
 * fold the last chunk's weights in.  Requires 0 <= S <= min(max_chunk, N_C),
 * 0 <= P and P + S < INT32_MAX. */
H2OKV_API int h2o_evict_insert(h2okv_cache *cache, const float *w_prev, const void *k_new,
                     const void *v_new, int32_t S, int64_t P, int32_t *slots_out,
                     void *stream);

/* h2o_evict_insert on n_caches caches at once: one pair of launches for every
 * (cache, b, h_k), for independent layers that advance chunk by chunk in step
 * (the layer loop of §A.5.1 run with every layer's chunk inputs at hand).
 * Host arrays of n_caches entries: caches (distinct handles that agree in
 * their description, fill level and score mode), w_prev (NULL array = no
 * fold; else every entry non-NULL), k_new, v_new, slots_out (NULL array, or
 * entries that may be NULL); each entry is what h2o_evict_insert takes for
 * that cache.  Same S and P for every cache.  On an argument error nothing is
 * enqueued; the caches' workspaces must not be in use by other calls. */
H2OKV_API int h2o_evict_insert_many(h2okv_cache *const *caches, int32_t n_caches,
                                    const float *const *w_prev, const void *const *k_new,
                                    const void *const *v_new, int32_t S, int64_t P,
                                    int32_t *const *slots_out, void *stream);

/* Score variant that ranks occupied slots in step 2 of h2o_evict_insert
 * ("Learning how to Forget", §3.1.1 Variants of Heavy-Hitter Oracle):
 *   H2OKV_SCORE_H2O       the cumulative score (default);
 *   H2OKV_SCORE_H2O_NORM  score / (t - token_pos) with t = P, the first
 *                         position of the chunk being inserted (the pages leave
 *                         t undefined; this is the reading used), computed as an
 *                         IEEE float32 quotient; an age below 1 counts as 1;
 *   H2OKV_SCORE_H2O_ORIG  the score summed over the batch rows (float32, in
 *                         batch order): every batch row evicts the same slots.
 * Empty slots are taken first in every variant.  Host only; applies to the
 * following calls. */
enum h2okv_score_mode { H2OKV_SCORE_H2O = 0, H2OKV_SCORE_H2O_NORM = 1, H2OKV_SCORE_H2O_ORIG = 2 };
H2OKV_API int kv_cache_set_score_mode(h2okv_cache *cache, int32_t mode);

/* Delta encoding of one update (§A.5.3: for keys' = scatter(keys, index,
 * key_new) it keeps delta_key = gather(keys, index), from which keys is rebuilt
 * as scatter(keys', index, delta_key)).  Caller-owned device buffers, indexed
 * like the chunk: keys, values [B, H_k, S, row bytes] in the cache's storage
 * format (bytes as stored: f32 / bf16 values, int8 codes, packed int4 codes),
 * k_scales, v_scales [B, H_k, S] fp16 (quantized caches, else NULL),
 * token_pos [B, H_k, S] int32 (the overwritten token positions; INT32_MAX for a
 * slot that was empty).  16-byte aligned. */
typedef struct h2okv_delta {
  void *keys;
  void *values;
  void *k_scales;
  void *v_scales;
  int32_t *token_pos;
} h2okv_delta;

/* h2o_evict_insert that also writes the delta encoding of the update: before
 * chunk row k overwrites its slot, the slot's stored key/value row, scales and
 * token position go to row k of `delta`.  slots_out is required (the index of
 * the delta encoding).  Same arguments and errors as h2o_evict_insert; S >= 1. */
H2OKV_API int h2o_evict_insert_delta(h2okv_cache *cache, const float *w_prev, const void *k_new,
                                     const void *v_new, int32_t S, int64_t P, int32_t *slots_out,
                                     const h2okv_delta *delta, void *stream);

/* Replay of logged eviction decisions (§3.2 / §A.5: a replay cache acts like
 * the cache, except that its decisions are read from the replay log):
 * step 1 of h2o_evict_insert, then chunk row k goes to slots_in[b, h_k, k]
 * (int32 [B, H_k, S], device) with token_pos = P + k and score 0.  The slots
 * of one (b, h_k) must be distinct; a slot outside [0, N_C) is skipped and
 * records H2OKV_ERR_INVALID_ARG in the device status word
 * (kv_cache_device_status).  delta may be NULL, else it receives the delta
 * encoding as in h2o_evict_insert_delta.  The fill level advances by S (capped
 * at N_C), as for a log written by a cache that filled left to right. */
H2OKV_API int h2o_insert_at(h2okv_cache *cache, const float *w_prev, const void *k_new,
                            const void *v_new, int32_t S, int64_t P, const int32_t *slots_in,
                            const h2okv_delta *delta, void *stream);

/* Undo one update from its delta encoding (the recurrence of §A.5.3 played
 * backwards): for every (b, h_k, k), the row, scales and token position of
 * delta row k go back into slot slots[b, h_k, k].  Scores and the fill level
 * are left as they are (set the fill level with kv_cache_set_fill).  Slots
 * outside [0, N_C) are skipped and record H2OKV_ERR_INVALID_ARG in the device
 * status word. */
H2OKV_API int kv_cache_restore(h2okv_cache *cache, const int32_t *slots, int32_t S,
                               const h2okv_delta *delta, void *stream);

/* Gradients of one chunk's SDPA over the cache (§A.5: autograd runs over each
 * chunk while the cache decisions are replayed; the cache policy itself is not
 * differentiated).  With p_ij = exp(q_i.k_j/sqrt(d) - lse_i) on the visible
 * slots (the mask of attn_chunk_with_scoresum), dP_ij = dy_i.v_j,
 * D_i = sum_j p_ij dP_ij and dS_ij = p_ij (dP_ij - D_i):
 *   dq_out[b,h,i]  = sum_j dS_ij k_j / sqrt(d)               [B, H_q, S, d] f32
 *   dk_out[b,g,j]  = sum_{h in g, i} dS_ij q_i / sqrt(d)     [B, H_k, N_C, d] f32
 *   dv_out[b,g,j]  = sum_{h in g, i} p_ij dy_i               [B, H_k, N_C, d] f32
 * with respect to the stored (dequantized) keys and values; the outputs are
 * overwritten.  q, dy: [B, H_q, S, d] in q_dtype; lse: [B, H_q, S] float32, the
 * natural-log row log-sum-exp written by attn_chunk_with_scoresum for the same
 * chunk and cache state.  The workspace holds D.  Same S / P rules as
 * attn_chunk_with_scoresum.  A bf16 cache with d_h = 128 and bf16 queries runs
 * on the tensor cores (three kernels on `stream`, the probabilities and dS
 * entering the second products as two bf16 terms each, hi + lo); every other
 * combination on CUDA cores.  Every output element is summed in a fixed order
 * (no atomics), so repeated calls give identical results. */
H2OKV_API int attn_chunk_backward(h2okv_cache *cache, const void *q, const void *dy,
                                  const float *lse, int32_t S, int64_t P, float *dq_out,
                                  float *dk_out, float *dv_out, void *stream);

/* SDPA of one chunk of queries against the cache, with summed weights (§A.1,
 * §A.7).  For query head h (group g = h / q_g), row i (token P + i):
 *   a_ij = q_i . k_j / sqrt(d_h), -inf where P + i < token_pos[b, g, j];
 *   m_ij = softmax_j(a_ij);  y_i = sum_j m_ij v_j;  lse_i = log sum_j exp(a_ij).
 * q:      [B, H_q, S, d_h] in q_dtype.         y_out: same shape and dtype.
 * lse_out:[B, H_q, S] float32, or NULL.
 * w_out:  [B, H_k, N_C] float32: sum over the chunk's rows and the group's
 *         q_g heads of m_ij (every slot written; unseen slots get 0).
 * wq_out: [B, H_q, N_C] float32 per-query-head sums, or NULL.
 * A row that sees no slot (cannot happen after h2o_evict_insert of the same
 * chunk) gets y = 0, lse = -inf and adds no weight.
 * Requires 1 <= S <= max_chunk, 0 <= P, P + S < INT32_MAX. */
H2OKV_API int attn_chunk_with_scoresum(h2okv_cache *cache, const void *q, int32_t S, int64_t P,
                             void *y_out, float *lse_out, float *w_out, float *wq_out,
                             void *stream);

/* Allocation-free variant of attn_chunk_with_scoresum (the paper has no
 * counterpart: it is an interface for callers that cannot allocate device
 * memory).  Some callers own no device allocations of their own -- every byte
 * they touch belongs to another allocator, such as a framework's caching pool
 * or an inference engine's fixed arena -- so they cannot provide the per-cache
 * workspace that kv_cache_create requires.  This call needs neither a handle
 * nor a workspace: it takes the cache description and buffers directly and
 * keeps its only scratch (one float32 log-sum-exp per query row) in a
 * file-scope device array inside the library.  It computes what
 * attn_chunk_with_scoresum computes, with the same arguments and layouts
 * (keys/values/scales/token_pos as in h2okv_cache_buffers; q, y_out, lse_out,
 * w_out, wq_out as in attn_chunk_with_scoresum), on the library's CUDA-core
 * kernels.
 *   - Limit: batch * n_q_heads * S <= 262144 rows (and batch * n_kv_heads <=
 *     65535); larger calls return H2OKV_ERR_INVALID_ARG without enqueuing
 *     anything.
 *   - The array (1 MiB) exists on every GPU that loads the library and is held
 *     until the process exits.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress)
 *     with the caller's device current, so the address always belongs to the
 *     current context.  The first call on a device also loads the library's
 *     device code there; make that first call before any stream capture.
 *   - Every call on a device shares the one array and leaves the last call's
 *     contents in it; calls whose work overlaps on the GPU (different streams,
 *     no ordering between them) race on it and give undefined results.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine. */
H2OKV_API int attn_chunk_with_scoresum_noalloc(const h2okv_cache_desc *desc, const void *keys,
                                               const void *values, const void *k_scales,
                                               const void *v_scales, const int32_t *token_pos,
                                               const void *q, int32_t S, int64_t P, void *y_out,
                                               float *lse_out, float *w_out, float *wq_out,
                                               void *stream);

/* Message of the last error on this thread ("" if none). */
H2OKV_API const char *h2okv_last_error(void);

/* Library ABI version (currently 1). */
H2OKV_API int32_t h2okv_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* H2OKV_H */
