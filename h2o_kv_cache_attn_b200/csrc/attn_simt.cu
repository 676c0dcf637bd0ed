// General CUDA-core path of chunked cache attention with summed weights
// ("Learning how to Forget", §A.1 token-position mask, §A.7 SDPA plus the
// attention weights summed over the query axis).  It serves every dtype and
// head dimension (float32 caches, head dimensions other than 128); the
// tensor-core path in attn_tc.cu takes bf16 / int8 / int4 caches with d = 128.
//
// Two passes over the cache per chunk:
//   pass 1  per packed query row: base-2 log-sum-exp over the visible slots
//           (online max / sum);
//   pass 2  p_ij = exp2(s_ij * log2(e) / sqrt(d) - lse2_i) with the FINAL
//           row statistics, so y = sum_j p_ij v_j needs no rescaling and the
//           column sums of p are the summed weights directly.
// Rows of the q_g query heads of one KV head are packed: packed row r of group
// g is head g*q_g + r / S, chunk row r % S.
#include <math.h>


#include "h2okv_internal.cuh"

namespace h2okv {
namespace {

constexpr int kRows = 32;    // packed query rows per CTA (8 warps x 4)
constexpr int kKeys = 32;    // slots per tile (one per lane)
constexpr int kThreads = 256;

template <int KV>
__device__ __forceinline__ float load_kv(const uint8_t *__restrict__ row, const __half *scale,
                                         int e) {
  if constexpr (KV == H2OKV_F32) {
    return reinterpret_cast<const float *>(row)[e];
  } else if constexpr (KV == H2OKV_BF16) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(row)[e]);
  } else if constexpr (KV == H2OKV_I8) {
    return (float)(int8_t)row[e] * __half2float(*scale);  // exact: 8-bit x 11-bit significand
  } else {
    const uint8_t b = row[e >> 1];
    int v = (e & 1) ? (b >> 4) : (b & 0xF);
    v = v >= 8 ? v - 16 : v;
    return (float)v * __half2float(*scale);
  }
}

template <int QT>
__device__ __forceinline__ float load_q(const void *q, size_t idx) {
  if constexpr (QT == H2OKV_F32)
    return reinterpret_cast<const float *>(q)[idx];
  else
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(q)[idx]);
}

struct SimtArgs {
  const void *q;
  const uint8_t *keys, *values;
  const __half *k_scales, *v_scales;
  const int32_t *token_pos;
  void *y;
  float *lse_out, *lse2, *w, *wq;
  int Hq, Hk, q_g, d, N_C, S, P;
  size_t row_bytes;
  float scale2;  // log2(e) / sqrt(d)
};

// Shared-memory carve-up (floats): q tile [kRows][d], k tile [kKeys][d+1],
// v tile [kKeys][d], p tile [kRows][kKeys+1], token_pos [kKeys], lse2 [kRows].
__host__ __device__ inline size_t simt_smem_bytes(int d) {
  return 4 * ((size_t)kRows * d + (size_t)kKeys * (d + 1) + (size_t)kKeys * d +
              (size_t)kRows * (kKeys + 1) + kKeys + kRows);
}

template <int QT, int KV, bool PASS2>
__global__ void __launch_bounds__(kThreads) simt_attn_kernel(SimtArgs a) {
  extern __shared__ float sm[];
  const int d = a.d;
  float *qs = sm;
  float *ks = qs + kRows * d;
  float *vs = ks + kKeys * (d + 1);
  float *ps = vs + kKeys * d;
  int *tps = reinterpret_cast<int *>(ps + kRows * (kKeys + 1));
  float *ls = reinterpret_cast<float *>(tps + kKeys);

  const int g_flat = blockIdx.y;  // b * Hk + g
  const int b = g_flat / a.Hk, g = g_flat - b * a.Hk;
  const int n_packed = a.q_g * a.S;
  const int r_begin = blockIdx.x * kRows;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // Stage the CTA's query rows (zeros past the end).
  for (int idx = tid; idx < kRows * d; idx += kThreads) {
    const int rr = idx / d, e = idx - rr * d;
    const int r = r_begin + rr;
    float v = 0.f;
    if (r < n_packed) {
      const int h = g * a.q_g + r / a.S, i = r % a.S;
      v = load_q<QT>(a.q, ((size_t)(b * a.Hq + h) * a.S + i) * d + e);
    }
    qs[idx] = v;
  }
  // Row metadata of this warp's 4 rows.
  int row_ok[4], row_i[4];
  size_t row_lin[4];  // (b*Hq + h)*S + i
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = r_begin + warp * 4 + rr;
    row_ok[rr] = r < n_packed;
    const int h = g * a.q_g + (row_ok[rr] ? r / a.S : 0);
    row_i[rr] = row_ok[rr] ? r % a.S : 0;
    row_lin[rr] = (size_t)(b * a.Hq + h) * a.S + row_i[rr];
  }
  if (PASS2) {
    if (tid < kRows) {
      const int r = r_begin + tid;
      float l = -INFINITY;
      if (r < n_packed) {
        const int h = g * a.q_g + r / a.S, i = r % a.S;
        l = a.lse2[(size_t)(b * a.Hq + h) * a.S + i];
      }
      ls[tid] = l;
    }
  }
  float m[4], l[4];
  constexpr int kMaxCols = kMaxHeadDim / 32;
  float o[4][kMaxCols];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxCols; ++c) o[rr][c] = 0.f;
  }
  const size_t slot0 = (size_t)g_flat * a.N_C;
  const uint8_t *kbase = a.keys + slot0 * a.row_bytes;
  const uint8_t *vbase = a.values + slot0 * a.row_bytes;
  const __half *ksc = a.k_scales ? a.k_scales + slot0 : nullptr;
  const __half *vsc = a.v_scales ? a.v_scales + slot0 : nullptr;
  const int32_t *tpb = a.token_pos + slot0;

  for (int t0 = 0; t0 < a.N_C; t0 += kKeys) {
    __syncthreads();  // previous tile fully consumed
    for (int idx = tid; idx < kKeys * d; idx += kThreads) {
      const int kk = idx / d, e = idx - kk * d;
      const int j = t0 + kk;
      float kv = 0.f, vv = 0.f;
      if (j < a.N_C) {
        kv = load_kv<KV>(kbase + (size_t)j * a.row_bytes, ksc ? ksc + j : nullptr, e);
        if (PASS2) vv = load_kv<KV>(vbase + (size_t)j * a.row_bytes, vsc ? vsc + j : nullptr, e);
      }
      ks[kk * (d + 1) + e] = kv;
      if (PASS2) vs[kk * d + e] = vv;
    }
    if (tid < kKeys) tps[tid] = (t0 + tid < a.N_C) ? tpb[t0 + tid] : kEmptyPos;
    __syncthreads();

    // logits: lane = slot of the tile, 4 rows per warp
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float *krow = ks + lane * (d + 1);
    const float *q0 = qs + (warp * 4) * d;
    for (int e = 0; e < d; ++e) {
      const float kv = krow[e];
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) acc[rr] = fmaf(q0[rr * d + e], kv, acc[rr]);
    }
    const int tpj = tps[lane];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const bool vis = row_ok[rr] && (int64_t)tpj <= (int64_t)a.P + row_i[rr];
      const float x = acc[rr] * a.scale2;
      if (!PASS2) {
        if (vis) {
          if (x > m[rr]) {
            l[rr] = l[rr] * exp2f(m[rr] - x) + 1.f;
            m[rr] = x;
          } else {
            l[rr] += exp2f(x - m[rr]);
          }
        }
      } else {
        const float lse2 = ls[warp * 4 + rr];
        const float p = (vis && lse2 != -INFINITY) ? exp2f(x - lse2) : 0.f;
        ps[(warp * 4 + rr) * (kKeys + 1) + lane] = p;
      }
    }
    if (PASS2) {
      __syncthreads();
      // summed weights: thread = slot; rows grouped by query head
      if (tid < kKeys && t0 + tid < a.N_C) {
        const int j = t0 + tid;
        float tot = 0.f, head_sum = 0.f;
        int cur_h = -1;
        for (int rr = 0; rr < kRows; ++rr) {
          const int r = r_begin + rr;
          if (r >= n_packed) break;
          const int hl = r / a.S;
          if (hl != cur_h) {
            if (cur_h >= 0 && a.wq && head_sum != 0.f)
              atomicAdd(a.wq + ((size_t)(b * a.Hq + g * a.q_g + cur_h)) * a.N_C + j, head_sum);
            cur_h = hl;
            head_sum = 0.f;
          }
          const float p = ps[rr * (kKeys + 1) + tid];
          head_sum += p;
          tot += p;
        }
        if (cur_h >= 0 && a.wq && head_sum != 0.f)
          atomicAdd(a.wq + ((size_t)(b * a.Hq + g * a.q_g + cur_h)) * a.N_C + j, head_sum);
        if (tot != 0.f) atomicAdd(a.w + (size_t)g_flat * a.N_C + j, tot);
      }
      // y += p v: lane owns columns lane, lane+32, ...
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const float *prow = ps + (warp * 4 + rr) * (kKeys + 1);
        for (int kk = 0; kk < kKeys; ++kk) {
          const float p = prow[kk];
          const float *vrow = vs + kk * d;
#pragma unroll
          for (int c = 0; c < kMaxCols; ++c) {
            const int e = lane + 32 * c;
            if (e < d) o[rr][c] = fmaf(p, vrow[e], o[rr][c]);
          }
        }
      }
    }
  }

  if (!PASS2) {
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      float M = m[rr];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
      float L = (M == -INFINITY) ? 0.f : l[rr] * exp2f(m[rr] - M);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
      if (lane == 0 && row_ok[rr]) {
        const float lse2 = (M == -INFINITY) ? -INFINITY : M + log2f(L);
        a.lse2[row_lin[rr]] = lse2;
        if (a.lse_out) a.lse_out[row_lin[rr]] = lse2 * 0.69314718055994531f;
      }
    }
  } else {
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      if (!row_ok[rr]) continue;
#pragma unroll
      for (int c = 0; c < kMaxCols; ++c) {
        const int e = lane + 32 * c;
        if (e >= d) continue;
        const size_t idx = row_lin[rr] * d + e;
        if (QT == H2OKV_F32)
          reinterpret_cast<float *>(a.y)[idx] = o[rr][c];
        else
          reinterpret_cast<__nv_bfloat16 *>(a.y)[idx] = __float2bfloat16_rn(o[rr][c]);
      }
    }
  }
}

template <int QT, int KV>
int run(SimtArgs &a, int B, cudaStream_t st) {
  const size_t smem = simt_smem_bytes(a.d);
  static thread_local int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    const int cap = (int)simt_smem_bytes(kMaxHeadDim);
    cudaError_t e1 = cudaFuncSetAttribute(simt_attn_kernel<QT, KV, false>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
    cudaError_t e2 = cudaFuncSetAttribute(simt_attn_kernel<QT, KV, true>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
    if (e1 != cudaSuccess || e2 != cudaSuccess)
      return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(simt_attn_kernel) failed");
    configured_dev = dev;
  }
  dim3 grid((a.q_g * a.S + kRows - 1) / kRows, B * a.Hk);
  simt_attn_kernel<QT, KV, false><<<grid, kThreads, smem, st>>>(a);
  int rc = check_launch("simt_attn_kernel pass 1");
  if (rc) return rc;
  simt_attn_kernel<QT, KV, true><<<grid, kThreads, smem, st>>>(a);
  return check_launch("simt_attn_kernel pass 2");
}

}  // namespace

// The CUDA-core grid (row tiles of one (batch row, KV head), B * H_k) must fit the launch
// limits; checked before anything is enqueued.
static int simt_grid_check(int B, int Hk, int q_g, int S) {
  const long long gx = ((long long)q_g * S + kRows - 1) / kRows;
  const long long gy = (long long)B * Hk;
  if (gy > 65535 || gx > INT32_MAX)
    return set_error(H2OKV_ERR_INVALID_ARG,
                     "batch * n_kv_heads = %lld (max 65535) or query rows per group too large", gy);
  return H2OKV_OK;
}

int launch_attn_simt(h2okv_cache *c, const void *q, int S, int64_t P, void *y, float *lse,
                     float *w, float *wq, cudaStream_t st) {
  const h2okv_cache_desc &d = c->desc;
  SimtArgs a;
  a.q = q;
  a.keys = reinterpret_cast<const uint8_t *>(c->bufs.keys);
  a.values = reinterpret_cast<const uint8_t *>(c->bufs.values);
  a.k_scales = reinterpret_cast<const __half *>(c->bufs.k_scales);
  a.v_scales = reinterpret_cast<const __half *>(c->bufs.v_scales);
  a.token_pos = c->bufs.token_pos;
  a.y = y;
  a.lse_out = lse;
  a.lse2 = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(c->bufs.workspace) + c->ws.lse2);
  a.w = w;
  a.wq = wq;
  a.Hq = d.n_q_heads;
  a.Hk = d.n_kv_heads;
  a.q_g = d.n_q_heads / d.n_kv_heads;
  a.d = d.head_dim;
  a.N_C = d.capacity;
  a.S = S;
  a.P = (int)P;
  a.row_bytes = c->row_bytes;
  a.scale2 = (float)(1.4426950408889634 / sqrt((double)d.head_dim));
  const int grc = simt_grid_check(d.batch, d.n_kv_heads, a.q_g, S);
  if (grc) return grc;

  const size_t nw = (size_t)d.batch * d.n_kv_heads * d.capacity * 4;
  if (cudaMemsetAsync(w, 0, nw, st) != cudaSuccess ||
      (wq && cudaMemsetAsync(wq, 0, nw * a.q_g, st) != cudaSuccess))
    return set_error(H2OKV_ERR_CUDA, "cudaMemsetAsync of w_out/wq_out failed");
  if (d.q_dtype == H2OKV_F32) return run<H2OKV_F32, H2OKV_F32>(a, d.batch, st);
  switch (d.kv_dtype) {
    case H2OKV_BF16: return run<H2OKV_BF16, H2OKV_BF16>(a, d.batch, st);
    case H2OKV_I8: return run<H2OKV_BF16, H2OKV_I8>(a, d.batch, st);
    case H2OKV_I4: return run<H2OKV_BF16, H2OKV_I4>(a, d.batch, st);
  }
  return set_error(H2OKV_ERR_UNSUPPORTED, "dtype combination");
}

}  // namespace h2okv

// ---- allocation-free entry point ---------------------------------------------------
// Some callers cannot allocate device memory: every byte they use is owned by
// another allocator (a framework's caching pool, an inference engine's fixed
// arena), so they cannot size and hand over the per-cache workspace that
// attn_chunk_with_scoresum needs.  attn_chunk_with_scoresum_noalloc runs the
// CUDA-core attention above with its only scratch -- one base-2 log-sum-exp per
// query row -- in a file-scope __device__ array instead.
namespace h2okv {
namespace {

// B * H_q * S rows the array holds (1 MiB of float per device).
constexpr size_t kNoAllocMaxRows = size_t(1) << 18;

static __device__ __align__(256) float g_noalloc_lse2[kNoAllocMaxRows];

// Device address of the array for the current device and context.  In host code the
// array's name is only a host-side stand-in, so the address is looked up, with the
// device current, on every call: a host-side query that allocates nothing, and that
// stays right if the context is torn down and made again (the module then loads at a
// new address).
int noalloc_scratch(float **out) {
  void *ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_lse2);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
  *out = static_cast<float *>(ptr);
  return H2OKV_OK;
}

}  // namespace
}  // namespace h2okv

extern "C" int attn_chunk_with_scoresum_noalloc(const h2okv_cache_desc *desc, const void *keys,
                                                const void *values, const void *k_scales,
                                                const void *v_scales, const int32_t *token_pos,
                                                const void *q, int32_t S, int64_t P, void *y_out,
                                                float *lse_out, float *w_out, float *wq_out,
                                                void *stream) {
  using namespace h2okv;
  set_error(H2OKV_OK, "");
  size_t sizes[H2OKV_NUM_BUFS];
  int rc = kv_cache_query_sizes(desc, sizes);  // validates the description
  if (rc) return rc;
  const bool quant = desc->kv_dtype == H2OKV_I8 || desc->kv_dtype == H2OKV_I4;
  if (!keys || !values || !token_pos || !q || !y_out || !w_out || (quant && (!k_scales || !v_scales)))
    return set_error(H2OKV_ERR_INVALID_ARG, "a required buffer is NULL");
  if (S < 1 || S > desc->max_chunk)
    return set_error(H2OKV_ERR_INVALID_ARG, "S = %d outside [1, max_chunk %d]", S,
                     desc->max_chunk);
  if (P < 0 || P + S >= (int64_t)INT32_MAX)
    return set_error(H2OKV_ERR_INVALID_ARG, "P = %lld out of range for int32 token positions",
                     (long long)P);
  const size_t rows = (size_t)desc->batch * desc->n_q_heads * S;
  if (rows > kNoAllocMaxRows)
    return set_error(H2OKV_ERR_INVALID_ARG,
                     "batch * n_q_heads * S = %zu exceeds the %zu rows of the static scratch", rows,
                     kNoAllocMaxRows);
  rc = simt_grid_check(desc->batch, desc->n_kv_heads, desc->n_q_heads / desc->n_kv_heads, S);
  if (rc) return rc;
  float *scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;

  cudaStream_t st = (cudaStream_t)stream;
  SimtArgs a;
  a.q = q;
  a.keys = reinterpret_cast<const uint8_t *>(keys);
  a.values = reinterpret_cast<const uint8_t *>(values);
  a.k_scales = quant ? reinterpret_cast<const __half *>(k_scales) : nullptr;
  a.v_scales = quant ? reinterpret_cast<const __half *>(v_scales) : nullptr;
  a.token_pos = token_pos;
  a.y = y_out;
  a.lse_out = lse_out;
  a.lse2 = scratch;  // fully written by pass 1 before pass 2 reads it: no clearing needed
  a.w = w_out;
  a.wq = wq_out;
  a.Hq = desc->n_q_heads;
  a.Hk = desc->n_kv_heads;
  a.q_g = desc->n_q_heads / desc->n_kv_heads;
  a.d = desc->head_dim;
  a.N_C = desc->capacity;
  a.S = S;
  a.P = (int)P;
  a.row_bytes = kv_row_bytes(desc->kv_dtype, desc->head_dim);
  a.scale2 = (float)(1.4426950408889634 / sqrt((double)desc->head_dim));
  const size_t nw = (size_t)desc->batch * desc->n_kv_heads * desc->capacity * 4;
  if (cudaMemsetAsync(w_out, 0, nw, st) != cudaSuccess ||
      (wq_out && cudaMemsetAsync(wq_out, 0, nw * a.q_g, st) != cudaSuccess))
    return set_error(H2OKV_ERR_CUDA, "cudaMemsetAsync of w_out/wq_out failed");
  if (desc->q_dtype == H2OKV_F32) return run<H2OKV_F32, H2OKV_F32>(a, desc->batch, st);
  switch (desc->kv_dtype) {
    case H2OKV_BF16: return run<H2OKV_BF16, H2OKV_BF16>(a, desc->batch, st);
    case H2OKV_I8: return run<H2OKV_BF16, H2OKV_I8>(a, desc->batch, st);
    case H2OKV_I4: return run<H2OKV_BF16, H2OKV_I4>(a, desc->batch, st);
  }
  return set_error(H2OKV_ERR_UNSUPPORTED, "dtype combination");
}
