// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "h2okv.h"

namespace h2okv {

constexpr int32_t kEmptyPos = INT32_MAX;
constexpr int kMaxHeadDim = 256;
constexpr int kMaxCapacity = 65536;

// Workspace carve-up of one cache (all offsets 256-byte aligned).
struct WorkspaceLayout {
  size_t lse2;         // float [B*Hq*max_chunk]: base-2 log-sum-exp per query row
  size_t part_ml;      // float2 [split CTAs * segments * 2 * 128]: partial (max, sum) per row
  size_t part_w;       // float [B*Hq*row_tiles*N_C]: per-row-tile summed weights (tensor-core path)
  size_t part_o;       // float [split CTAs * segments * 2 * 128 * d]: partial outputs
  size_t nlse;         // float [B*Hq*row_tiles*128]: -lse2 per row of every row tile
  size_t status;       // int32: device status word (0 = ok, else an H2OKV_ERR_* code)
  size_t ev_hist;      // uint32 [B*H_k][2048]: top-bit key histograms of the eviction (zero between calls)
  size_t ev_arrive;    // uint32 [B*H_k]: arrival counters of the eviction (zero between calls)
  size_t ev_slots;     // int32 [B*H_k][max_chunk]: chosen slots in slot order (zeroed on create
                       //   and reset, so a list a timed-out choose left unfinished stays in range)
  size_t ev_zero_end;  // [ev_hist, ev_zero_end) is zeroed on create and reset
  size_t total;
};

struct TcPlan {          // launch plan of the tensor-core path
  bool enabled;
  int tiles_per_head;    // ceil(max_chunk / 128)
  int split_ctas;        // CTAs of the split (persistent) kernels, 0 = split scheduling off
  int max_seg;           // segments per CTA the split workspace is sized for
  bool two_pass;         // bf16: attention pass + score-sum pass (else the fused kernel)
  int sms;               // multiprocessors of the device (0 if unknown)
  bool maps_ready;       // k_map / v_map encoded
  alignas(64) unsigned char k_map[128];  // CUtensorMap over keys
  alignas(64) unsigned char v_map[128];  // CUtensorMap over values
};

constexpr uint64_t kDefaultWaitTimeoutNs = 2000000000ull;  // bounded device waits

}  // namespace h2okv

struct h2okv_cache {
  h2okv_cache_desc desc;
  h2okv_cache_buffers bufs;
  int32_t n_filled;
  int32_t n_span;  // every slot at or past this index is empty (the attention scans [0, n_span))
  size_t row_bytes;  // bytes of one stored key/value row
  h2okv::WorkspaceLayout ws;
  h2okv::TcPlan tc;
  uint64_t wait_timeout_ns;
  int32_t score_mode;  // h2okv_score_mode
  int32_t sms;         // multiprocessors of the device the cache was created on (0 if unknown)
};

namespace h2okv {

// Error reporting (thread-local message).
int set_error(int code, const char *fmt, ...);
int check_launch(const char *what);

inline size_t kv_row_bytes(int kv_dtype, int d) {
  switch (kv_dtype) {
    case H2OKV_F32: return (size_t)d * 4;
    case H2OKV_BF16: return (size_t)d * 2;
    case H2OKV_I8: return (size_t)d;
    case H2OKV_I4: return (size_t)d / 2;
  }
  return 0;
}

// ---- launchers (return H2OKV_OK or an error code) -------------------------
int launch_init_cache(h2okv_cache *c, cudaStream_t st);
int launch_evict_insert(h2okv_cache *c, const float *w_prev, const void *k_new, const void *v_new,
                        int S, int64_t P, int32_t *slots_out, const int32_t *slots_in,
                        const h2okv_delta *delta, cudaStream_t st);
int launch_evict_insert_many(h2okv_cache *const *caches, int n, const float *const *w_prev,
                             const void *const *k_new, const void *const *v_new, int S, int64_t P,
                             int32_t *const *slots_out, cudaStream_t st);
int launch_restore(h2okv_cache *c, const int32_t *slots, int S, const h2okv_delta *delta,
                   cudaStream_t st);
int launch_attn_backward(h2okv_cache *c, const void *q, const void *dy, const float *lse, int S,
                         int64_t P, float *dq, float *dk, float *dv, cudaStream_t st);
int launch_quantize(int kv_dtype, const __nv_bfloat16 *x, int64_t n_rows, int d, void *codes,
                    __half *scales, cudaStream_t st);
int launch_attn_simt(h2okv_cache *c, const void *q, int S, int64_t P, void *y, float *lse,
                     float *w, float *wq, cudaStream_t st);
bool tc_path_supported(const h2okv_cache_desc &d);
int launch_attn_tc(h2okv_cache *c, const void *q, int S, int64_t P, void *y, float *lse, float *w,
                   float *wq, cudaStream_t st);
void tc_plan(const h2okv_cache_desc &d, TcPlan *plan);
// 3-D bf16 tensor map over [planes][rows][128] with a (64 x 128 x 1) box, 128-byte swizzle.
int encode_rows_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t planes);
// The cache's key / value tensor maps (bf16 caches), encoded once.
int ensure_cache_maps(h2okv_cache *c);
bool bwd_tc_supported(const h2okv_cache_desc &d);
int launch_attn_backward_tc(h2okv_cache *c, const void *q, const void *dy, const float *lse, int S,
                            int64_t P, float *dq, float *dk, float *dv, cudaStream_t st);

}  // namespace h2okv
