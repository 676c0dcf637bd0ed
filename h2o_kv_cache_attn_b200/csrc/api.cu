// C ABI entry points: argument validation, buffer sizing and dispatch to the
// kernels.  Every check runs on the host before anything is enqueued.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "h2okv_internal.cuh"

namespace h2okv {

static thread_local char g_err[512];

int set_error(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int check_launch(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return H2OKV_OK;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static int validate_desc(const h2okv_cache_desc *d) {
  if (!d) return set_error(H2OKV_ERR_INVALID_ARG, "desc is NULL");
  if (d->batch < 1 || d->n_kv_heads < 1 || d->n_q_heads < 1)
    return set_error(H2OKV_ERR_INVALID_ARG, "batch, n_q_heads and n_kv_heads must be >= 1");
  if (d->n_q_heads % d->n_kv_heads)
    return set_error(H2OKV_ERR_INVALID_ARG, "n_q_heads (%d) must be a multiple of n_kv_heads (%d)",
                     d->n_q_heads, d->n_kv_heads);
  if (d->head_dim < 8 || d->head_dim > kMaxHeadDim || d->head_dim % 8)
    return set_error(H2OKV_ERR_INVALID_ARG, "head_dim %d must be a multiple of 8 in [8, %d]",
                     d->head_dim, kMaxHeadDim);
  if (d->capacity < 1 || d->capacity > kMaxCapacity)
    return set_error(H2OKV_ERR_INVALID_ARG, "capacity %d must be in [1, %d]", d->capacity,
                     kMaxCapacity);
  if (d->max_chunk < 1)
    return set_error(H2OKV_ERR_INVALID_ARG, "max_chunk must be >= 1");
  if (d->q_dtype != H2OKV_F32 && d->q_dtype != H2OKV_BF16)
    return set_error(H2OKV_ERR_INVALID_ARG, "q_dtype must be F32 or BF16");
  switch (d->kv_dtype) {
    case H2OKV_F32:
      if (d->q_dtype != H2OKV_F32)
        return set_error(H2OKV_ERR_INVALID_ARG, "an F32 cache needs q_dtype F32");
      break;
    case H2OKV_BF16:
    case H2OKV_I8:
    case H2OKV_I4:
      if (d->q_dtype != H2OKV_BF16)
        return set_error(H2OKV_ERR_INVALID_ARG, "BF16/I8/I4 caches need q_dtype BF16");
      break;
    default:
      return set_error(H2OKV_ERR_INVALID_ARG, "unknown kv_dtype %d", d->kv_dtype);
  }
  const int64_t rows = (int64_t)d->batch * d->n_q_heads * d->max_chunk;
  if (rows > (int64_t)1 << 31)
    return set_error(H2OKV_ERR_INVALID_ARG, "batch * n_q_heads * max_chunk too large");
  return H2OKV_OK;
}

static void layout(const h2okv_cache_desc &d, const TcPlan &tc, WorkspaceLayout *ws) {
  const size_t B = d.batch, Hq = d.n_q_heads, NC = d.capacity, S = d.max_chunk,
               D = d.head_dim;
  size_t off = 0;
  ws->lse2 = off;
  off = align256(off + B * Hq * S * 4);
  ws->status = off;
  off = align256(off + 4);
  const size_t G = (size_t)d.batch * d.n_kv_heads;
  ws->ev_hist = off;
  off = align256(off + G * 2048 * 4);
  ws->ev_arrive = off;
  off = align256(off + G * 4);
  ws->ev_slots = off;
  off = align256(off + G * S * 4);
  ws->ev_zero_end = off;
  ws->part_ml = ws->part_w = ws->part_o = ws->nlse = off;
  if (tc.enabled) {
    const size_t seg_rows = (size_t)tc.split_ctas * tc.max_seg * 2 * 128;
    ws->part_ml = off;
    off = align256(off + seg_rows * 8);
    ws->part_w = off;
    off = align256(off + B * Hq * (size_t)tc.tiles_per_head * NC * 4);
    ws->part_o = off;
    off = align256(off + seg_rows * D * 4);
    ws->nlse = off;
    off = align256(off + B * Hq * (size_t)tc.tiles_per_head * 128 * 4);
  }
  ws->total = off;
}

static void sizes_of(const h2okv_cache_desc &d, const WorkspaceLayout &ws, size_t *sz) {
  const size_t slots = (size_t)d.batch * d.n_kv_heads * d.capacity;
  const size_t rb = kv_row_bytes(d.kv_dtype, d.head_dim);
  const bool quant = d.kv_dtype == H2OKV_I8 || d.kv_dtype == H2OKV_I4;
  sz[H2OKV_BUF_KEYS] = slots * rb;
  sz[H2OKV_BUF_VALUES] = slots * rb;
  sz[H2OKV_BUF_K_SCALES] = quant ? slots * 2 : 0;
  sz[H2OKV_BUF_V_SCALES] = quant ? slots * 2 : 0;
  sz[H2OKV_BUF_TOKEN_POS] = slots * 4;
  sz[H2OKV_BUF_SCORES] = slots * 4;
  sz[H2OKV_BUF_WORKSPACE] = ws.total;
}

static bool misaligned(const void *p, size_t a) { return ((uintptr_t)p) % a != 0; }

}  // namespace h2okv

using namespace h2okv;

extern "C" {

int32_t h2okv_abi_version(void) { return 1; }

const char *h2okv_last_error(void) { return g_err; }

int kv_cache_query_sizes(const h2okv_cache_desc *desc, size_t sizes[H2OKV_NUM_BUFS]) {
  g_err[0] = 0;
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (!sizes) return set_error(H2OKV_ERR_INVALID_ARG, "sizes is NULL");
  TcPlan tc;
  tc_plan(*desc, &tc);
  WorkspaceLayout ws;
  layout(*desc, tc, &ws);
  sizes_of(*desc, ws, sizes);
  return H2OKV_OK;
}

int kv_cache_create(const h2okv_cache_desc *desc, const h2okv_cache_buffers *bufs, void *stream,
                    h2okv_cache **out) {
  g_err[0] = 0;
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (!bufs || !out) return set_error(H2OKV_ERR_INVALID_ARG, "bufs/out is NULL");
  const bool quant = desc->kv_dtype == H2OKV_I8 || desc->kv_dtype == H2OKV_I4;
  if (!bufs->keys || !bufs->values || !bufs->token_pos || !bufs->scores || !bufs->workspace)
    return set_error(H2OKV_ERR_INVALID_ARG, "keys, values, token_pos, scores, workspace required");
  if (quant && (!bufs->k_scales || !bufs->v_scales))
    return set_error(H2OKV_ERR_INVALID_ARG, "I8/I4 caches need k_scales and v_scales");
  if (misaligned(bufs->keys, 16) || misaligned(bufs->values, 16) ||
      misaligned(bufs->workspace, 256) || misaligned(bufs->token_pos, 16) ||
      misaligned(bufs->scores, 16) || (quant && (misaligned(bufs->k_scales, 16) ||
                                                 misaligned(bufs->v_scales, 16))))
    return set_error(H2OKV_ERR_INVALID_ARG,
                     "buffers must be 16-byte aligned (workspace 256-byte aligned)");
  h2okv_cache *c = new (std::nothrow) h2okv_cache;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "out of host memory");
  c->desc = *desc;
  c->bufs = *bufs;
  if (!quant) c->bufs.k_scales = c->bufs.v_scales = nullptr;
  c->n_filled = 0;
  c->n_span = 0;
  c->row_bytes = kv_row_bytes(desc->kv_dtype, desc->head_dim);
  tc_plan(*desc, &c->tc);
  c->tc.maps_ready = false;
  c->wait_timeout_ns = kDefaultWaitTimeoutNs;
  c->score_mode = H2OKV_SCORE_H2O;
  {
    int dev = 0, sms = 0;
    c->sms = (cudaGetDevice(&dev) == cudaSuccess &&
              cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
                 ? sms
                 : 0;
    cudaGetLastError();
  }
  layout(*desc, c->tc, &c->ws);
  // The attention kernels read every slot and mask the empty ones arithmetically,
  // which needs finite values there: start from zeroed rows and scales.
  {
    const size_t n_slots = (size_t)desc->batch * desc->n_kv_heads * desc->capacity;
    cudaStream_t st = (cudaStream_t)stream;
    bool ok = cudaMemsetAsync(bufs->keys, 0, n_slots * c->row_bytes, st) == cudaSuccess &&
              cudaMemsetAsync(bufs->values, 0, n_slots * c->row_bytes, st) == cudaSuccess;
    if (ok && c->bufs.k_scales && c->bufs.v_scales)
      ok = cudaMemsetAsync(c->bufs.k_scales, 0, n_slots * 2, st) == cudaSuccess &&
           cudaMemsetAsync(c->bufs.v_scales, 0, n_slots * 2, st) == cudaSuccess;
    if (!ok) {
      delete c;
      return set_error(H2OKV_ERR_CUDA, "cudaMemsetAsync(cache rows) failed");
    }
  }
  rc = launch_init_cache(c, (cudaStream_t)stream);
  if (rc) {
    delete c;
    return rc;
  }
  *out = c;
  return H2OKV_OK;
}

int kv_cache_reset(h2okv_cache *c, void *stream) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  int rc = launch_init_cache(c, (cudaStream_t)stream);
  if (rc) return rc;
  c->n_filled = 0;
  c->n_span = 0;
  return H2OKV_OK;
}

int kv_cache_device_status(h2okv_cache *c, int32_t *status, void *stream) {
  g_err[0] = 0;
  if (!c || !status) return set_error(H2OKV_ERR_INVALID_ARG, "NULL argument");
  cudaStream_t st = (cudaStream_t)stream;
  int32_t *dev = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(c->bufs.workspace) +
                                             c->ws.status);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, dev, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(dev, 0, 4, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "reading the device status word failed: %s",
                     cudaGetErrorString(cudaGetLastError()));
  *status = v;
  return H2OKV_OK;
}

int kv_cache_set_wait_timeout(h2okv_cache *c, uint64_t timeout_ns) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  c->wait_timeout_ns = timeout_ns;
  return H2OKV_OK;
}

int kv_cache_destroy(h2okv_cache *c) {
  delete c;
  return H2OKV_OK;
}

int kv_cache_get_fill(const h2okv_cache *c, int32_t *n_filled) {
  g_err[0] = 0;
  if (!c || !n_filled) return set_error(H2OKV_ERR_INVALID_ARG, "NULL argument");
  *n_filled = c->n_filled;
  return H2OKV_OK;
}

int kv_cache_set_fill(h2okv_cache *c, int32_t n_filled) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  if (n_filled < 0 || n_filled > c->desc.capacity)
    return set_error(H2OKV_ERR_INVALID_ARG, "n_filled %d outside [0, %d]", n_filled,
                     c->desc.capacity);
  c->n_filled = n_filled;
  c->n_span = c->desc.capacity;  // a state written directly may occupy any slot
  return H2OKV_OK;
}

int kv_cache_quantize(int32_t kv_dtype, const void *x_bf16, int64_t n_rows, int32_t head_dim,
                      void *codes_out, void *scales_out, void *stream) {
  g_err[0] = 0;
  if (kv_dtype != H2OKV_I8 && kv_dtype != H2OKV_I4)
    return set_error(H2OKV_ERR_INVALID_ARG, "kv_dtype must be I8 or I4");
  if (head_dim < 8 || head_dim > kMaxHeadDim || head_dim % 8)
    return set_error(H2OKV_ERR_INVALID_ARG, "head_dim %d must be a multiple of 8 in [8, %d]",
                     head_dim, kMaxHeadDim);
  if (n_rows < 0) return set_error(H2OKV_ERR_INVALID_ARG, "n_rows < 0");
  if (n_rows == 0) return H2OKV_OK;
  if (!x_bf16 || !codes_out || !scales_out)
    return set_error(H2OKV_ERR_INVALID_ARG, "NULL buffer");
  if (n_rows > ((int64_t)1 << 40)) return set_error(H2OKV_ERR_INVALID_ARG, "n_rows too large");
  return launch_quantize(kv_dtype, (const __nv_bfloat16 *)x_bf16, n_rows, head_dim, codes_out,
                         (__half *)scales_out, (cudaStream_t)stream);
}

int h2o_evict_insert(h2okv_cache *c, const float *w_prev, const void *k_new, const void *v_new,
                     int32_t S, int64_t P, int32_t *slots_out, void *stream) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  if (S < 0 || S > c->desc.max_chunk || S > c->desc.capacity)
    return set_error(H2OKV_ERR_INVALID_ARG, "S = %d outside [0, min(max_chunk %d, capacity %d)]",
                     S, c->desc.max_chunk, c->desc.capacity);
  if (P < 0 || P + S >= (int64_t)INT32_MAX)
    return set_error(H2OKV_ERR_INVALID_ARG, "P = %lld out of range for int32 token positions",
                     (long long)P);
  if (S > 0 && (!k_new || !v_new))
    return set_error(H2OKV_ERR_INVALID_ARG, "k_new and v_new are required when S > 0");
  if (misaligned(k_new, 16) || misaligned(v_new, 16) || misaligned(w_prev, 4))
    return set_error(H2OKV_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
  if (S == 0 && !w_prev) return H2OKV_OK;
  int rc = launch_evict_insert(c, w_prev, k_new, v_new, S, P, slots_out, nullptr, nullptr,
                               (cudaStream_t)stream);
  if (rc) return rc;
  c->n_filled = c->n_filled + S > c->desc.capacity ? c->desc.capacity : c->n_filled + S;
  // the policy fills slots left to right before it evicts
  if (c->n_filled > c->n_span) c->n_span = c->n_filled;
  return H2OKV_OK;
}

int h2o_evict_insert_many(h2okv_cache *const *caches, int32_t n_caches,
                          const float *const *w_prev, const void *const *k_new,
                          const void *const *v_new, int32_t S, int64_t P,
                          int32_t *const *slots_out, void *stream) {
  g_err[0] = 0;
  if (!caches || n_caches < 1) return set_error(H2OKV_ERR_INVALID_ARG, "no caches");
  const h2okv_cache *c0 = caches[0];
  if (!c0) return set_error(H2OKV_ERR_INVALID_ARG, "cache 0 is NULL");
  if (S < 0 || S > c0->desc.max_chunk || S > c0->desc.capacity)
    return set_error(H2OKV_ERR_INVALID_ARG, "S = %d outside [0, min(max_chunk %d, capacity %d)]",
                     S, c0->desc.max_chunk, c0->desc.capacity);
  if (P < 0 || P + S >= (int64_t)INT32_MAX)
    return set_error(H2OKV_ERR_INVALID_ARG, "P = %lld out of range for int32 token positions",
                     (long long)P);
  if (S > 0 && (!k_new || !v_new))
    return set_error(H2OKV_ERR_INVALID_ARG, "k_new and v_new are required when S > 0");
  for (int i = 0; i < n_caches; ++i) {
    const h2okv_cache *c = caches[i];
    if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache %d is NULL", i);
    if (memcmp(&c->desc, &c0->desc, sizeof(c0->desc)) != 0 || c->n_filled != c0->n_filled ||
        c->score_mode != c0->score_mode)
      return set_error(H2OKV_ERR_INVALID_ARG,
                       "cache %d differs from cache 0 in shape, fill level or score mode", i);
    for (int j = 0; j < i; ++j)
      if (caches[j] == c) return set_error(H2OKV_ERR_INVALID_ARG, "cache %d is listed twice", i);
    if (S > 0 && (!k_new[i] || !v_new[i]))
      return set_error(H2OKV_ERR_INVALID_ARG, "k_new[%d] / v_new[%d] is NULL", i, i);
    if (S > 0 && (misaligned(k_new[i], 16) || misaligned(v_new[i], 16)))
      return set_error(H2OKV_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
    if (w_prev && (!w_prev[i] || misaligned(w_prev[i], 4)))
      return set_error(H2OKV_ERR_INVALID_ARG, "w_prev[%d] is NULL or misaligned", i);
  }
  if (S == 0 && !w_prev) return H2OKV_OK;
  int rc = launch_evict_insert_many(caches, n_caches, w_prev, k_new, v_new, S, P, slots_out,
                                    (cudaStream_t)stream);
  if (rc) return rc;
  for (int i = 0; i < n_caches; ++i) {
    h2okv_cache *c = caches[i];
    c->n_filled = c->n_filled + S > c->desc.capacity ? c->desc.capacity : c->n_filled + S;
    if (c->n_filled > c->n_span) c->n_span = c->n_filled;
  }
  return H2OKV_OK;
}

int kv_cache_set_score_mode(h2okv_cache *c, int32_t mode) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  if (mode != H2OKV_SCORE_H2O && mode != H2OKV_SCORE_H2O_NORM && mode != H2OKV_SCORE_H2O_ORIG)
    return set_error(H2OKV_ERR_INVALID_ARG, "unknown score mode %d", mode);
  c->score_mode = mode;
  return H2OKV_OK;
}

// Delta buffers: rows, token positions, and scales for quantized caches.
static int check_delta(const h2okv_cache *c, const h2okv_delta *dl) {
  if (!dl || !dl->keys || !dl->values || !dl->token_pos)
    return set_error(H2OKV_ERR_INVALID_ARG, "delta keys, values and token_pos are required");
  const bool quant = c->desc.kv_dtype == H2OKV_I8 || c->desc.kv_dtype == H2OKV_I4;
  if (quant && (!dl->k_scales || !dl->v_scales))
    return set_error(H2OKV_ERR_INVALID_ARG, "delta scales are required for I8/I4 caches");
  if (misaligned(dl->keys, 16) || misaligned(dl->values, 16) || misaligned(dl->token_pos, 16) ||
      (quant && (misaligned(dl->k_scales, 16) || misaligned(dl->v_scales, 16))))
    return set_error(H2OKV_ERR_INVALID_ARG, "delta buffers must be 16-byte aligned");
  return H2OKV_OK;
}

static int check_chunk(const h2okv_cache *c, const void *k_new, const void *v_new, int32_t S,
                       int64_t P, const float *w_prev) {
  if (S < 1 || S > c->desc.max_chunk || S > c->desc.capacity)
    return set_error(H2OKV_ERR_INVALID_ARG, "S = %d outside [1, min(max_chunk %d, capacity %d)]",
                     S, c->desc.max_chunk, c->desc.capacity);
  if (P < 0 || P + S >= (int64_t)INT32_MAX)
    return set_error(H2OKV_ERR_INVALID_ARG, "P = %lld out of range for int32 token positions",
                     (long long)P);
  if (!k_new || !v_new) return set_error(H2OKV_ERR_INVALID_ARG, "k_new and v_new are required");
  if (misaligned(k_new, 16) || misaligned(v_new, 16) || misaligned(w_prev, 4))
    return set_error(H2OKV_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
  return H2OKV_OK;
}

int h2o_evict_insert_delta(h2okv_cache *c, const float *w_prev, const void *k_new,
                           const void *v_new, int32_t S, int64_t P, int32_t *slots_out,
                           const h2okv_delta *delta, void *stream) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  int rc = check_chunk(c, k_new, v_new, S, P, w_prev);
  if (rc) return rc;
  if (!slots_out) return set_error(H2OKV_ERR_INVALID_ARG, "slots_out is required with a delta");
  rc = check_delta(c, delta);
  if (rc) return rc;
  rc = launch_evict_insert(c, w_prev, k_new, v_new, S, P, slots_out, nullptr, delta,
                           (cudaStream_t)stream);
  if (rc) return rc;
  c->n_filled = c->n_filled + S > c->desc.capacity ? c->desc.capacity : c->n_filled + S;
  if (c->n_filled > c->n_span) c->n_span = c->n_filled;
  return H2OKV_OK;
}

int h2o_insert_at(h2okv_cache *c, const float *w_prev, const void *k_new, const void *v_new,
                  int32_t S, int64_t P, const int32_t *slots_in, const h2okv_delta *delta,
                  void *stream) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  int rc = check_chunk(c, k_new, v_new, S, P, w_prev);
  if (rc) return rc;
  if (!slots_in) return set_error(H2OKV_ERR_INVALID_ARG, "slots_in is required");
  if (delta) {
    rc = check_delta(c, delta);
    if (rc) return rc;
  }
  rc = launch_evict_insert(c, w_prev, k_new, v_new, S, P, nullptr, slots_in, delta,
                           (cudaStream_t)stream);
  if (rc) return rc;
  c->n_filled = c->n_filled + S > c->desc.capacity ? c->desc.capacity : c->n_filled + S;
  c->n_span = c->desc.capacity;  // logged slots may lie anywhere
  return H2OKV_OK;
}

int kv_cache_restore(h2okv_cache *c, const int32_t *slots, int32_t S, const h2okv_delta *delta,
                     void *stream) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  if (S < 0 || S > c->desc.max_chunk || S > c->desc.capacity)
    return set_error(H2OKV_ERR_INVALID_ARG, "S = %d outside [0, min(max_chunk, capacity)]", S);
  if (S == 0) return H2OKV_OK;
  if (!slots) return set_error(H2OKV_ERR_INVALID_ARG, "slots is required");
  int rc = check_delta(c, delta);
  if (rc) return rc;
  return launch_restore(c, slots, S, delta, (cudaStream_t)stream);
}

int attn_chunk_backward(h2okv_cache *c, const void *q, const void *dy, const float *lse, int32_t S,
                        int64_t P, float *dq_out, float *dk_out, float *dv_out, void *stream) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  if (S < 1 || S > c->desc.max_chunk)
    return set_error(H2OKV_ERR_INVALID_ARG, "S = %d outside [1, max_chunk %d]", S,
                     c->desc.max_chunk);
  if (P < 0 || P + S >= (int64_t)INT32_MAX)
    return set_error(H2OKV_ERR_INVALID_ARG, "P = %lld out of range for int32 token positions",
                     (long long)P);
  if (!q || !dy || !lse || !dq_out || !dk_out || !dv_out)
    return set_error(H2OKV_ERR_INVALID_ARG, "q, dy, lse, dq_out, dk_out and dv_out are required");
  if (misaligned(q, 16) || misaligned(dy, 16) || misaligned(lse, 4) || misaligned(dq_out, 16) ||
      misaligned(dk_out, 16) || misaligned(dv_out, 16))
    return set_error(H2OKV_ERR_INVALID_ARG, "q, dy and the outputs must be 16-byte aligned");
  return launch_attn_backward(c, q, dy, lse, S, P, dq_out, dk_out, dv_out, (cudaStream_t)stream);
}

int attn_chunk_with_scoresum(h2okv_cache *c, const void *q, int32_t S, int64_t P, void *y_out,
                             float *lse_out, float *w_out, float *wq_out, void *stream) {
  g_err[0] = 0;
  if (!c) return set_error(H2OKV_ERR_INVALID_ARG, "cache is NULL");
  if (S < 1 || S > c->desc.max_chunk)
    return set_error(H2OKV_ERR_INVALID_ARG, "S = %d outside [1, max_chunk %d]", S,
                     c->desc.max_chunk);
  if (P < 0 || P + S >= (int64_t)INT32_MAX)
    return set_error(H2OKV_ERR_INVALID_ARG, "P = %lld out of range for int32 token positions",
                     (long long)P);
  if (!q || !y_out || !w_out)
    return set_error(H2OKV_ERR_INVALID_ARG, "q, y_out and w_out are required");
  if (misaligned(q, 16) || misaligned(y_out, 16) || misaligned(w_out, 16) ||
      (wq_out && misaligned(wq_out, 16)) || (lse_out && misaligned(lse_out, 4)))
    return set_error(H2OKV_ERR_INVALID_ARG, "q, y_out, w_out, wq_out must be 16-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  if (c->tc.enabled && S <= c->desc.max_chunk)
    return launch_attn_tc(c, q, S, P, y_out, lse_out, w_out, wq_out, st);
  return launch_attn_simt(c, q, S, P, y_out, lse_out, w_out, wq_out, st);
}

}  // extern "C"
