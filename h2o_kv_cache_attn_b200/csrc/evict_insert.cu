// H2O score update, lowest-score slot selection and overwrite of the chosen
// slots ("Learning how to Forget", §3.1 cache filled left to right then a
// per-(b, h) policy; §3.1.1 cumulative H2O score, lowest score evicted;
// §A.5.3 keys' = scatter(keys, index, key_new)), plus the 8/4-bit row
// quantizer used on insert.
//
// Two kernels per call:
//   select_kernel  one CTA per (b, h_k): scores += w_prev, then the S slots to
//                  overwrite -- empty slots first, then the smallest (score,
//                  slot) pairs -- by a 4-pass 8-bit radix select on
//                  order-preserving uint32 keys held in shared memory, and a
//                  block scan in slot order that lists the chosen slots
//                  ascending (token k -> k-th smallest slot);
//   scatter_kernel one warp per (b, h_k, k): copies (or quantizes) the new key
//                  and value rows into their slots.
// The quantizer must agree bit for bit with an IEEE float32 reference: it uses
// correctly rounded division, rintf and __float2half_rn only (this file is
// never built with fast-math).
#include "h2okv_internal.cuh"

namespace h2okv {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSmemKeyCap = 53248;  // keys held in shared memory up to this capacity

// Unsigned key with the order of the float: -0 and +0 map to the same key;
// every non-NaN score maps to a key >= 1 so that 0 can mark an empty slot.
__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7fffffffu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of one uint32 per thread (blockDim.x == kSelThreads).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_tot,
                                                         uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t wv = warp_tot[lane];
    uint32_t wincl = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t t = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += t;
    }
    warp_tot[lane] = wincl - wv;
    if (lane == 31) *total = wincl;
  }
  __syncthreads();
  uint32_t r = warp_tot[warp] + incl - v;
  __syncthreads();  // warp_tot is reused by the next call
  return r;
}

// mode 0: accumulate only; 1: fill slots n_filled.. (no occupied slot is
// touched); 2: generic selection (empty slots first, then lowest scores).
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(float *__restrict__ scores, const float *__restrict__ w_prev,
                  int32_t *__restrict__ token_pos, int N_C, int S, int P, int mode, int n_filled,
                  int max_chunk, int32_t *__restrict__ slot_list, int32_t *__restrict__ slots_out,
                  uint32_t *__restrict__ gkeys) {
  extern __shared__ uint32_t smem_keys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t s_prefix, s_k, s_total;

  const int bh = blockIdx.x;
  const size_t base = (size_t)bh * N_C;
  float *sc = scores + base;
  const float *wp = w_prev ? w_prev + base : nullptr;
  int32_t *tp = token_pos + base;
  uint32_t *keys = gkeys ? gkeys + base : smem_keys;
  int32_t *list = slot_list + (size_t)bh * max_chunk;
  int32_t *sout = slots_out ? slots_out + (size_t)bh * S : nullptr;
  const int tid = threadIdx.x, lane = tid & 31;

  // 1. scores += w_prev (float32), selection keys.
  for (int j = tid; j < N_C; j += blockDim.x) {
    float s = sc[j];
    if (wp) {
      s = __fadd_rn(s, wp[j]);
      sc[j] = s;
    }
    if (mode == 2) keys[j] = (tp[j] == kEmptyPos) ? 0u : order_key(s);
  }
  if (mode == 0) return;
  __syncthreads();
  if (mode == 1) {
    for (int k = tid; k < S; k += blockDim.x) {
      const int j = n_filled + k;
      list[k] = j;
      if (sout) sout[k] = j;
      tp[j] = P + k;
      sc[j] = 0.f;
    }
    return;
  }

  // 2. radix select of the S-th smallest key, 8 bits per pass from the top.
  uint32_t prefix = 0u, pmask = 0u, k = (uint32_t)S;
  const int n_round = (N_C + kSelThreads - 1) / kSelThreads;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (int r = 0; r < n_round; ++r) {
      const int j = r * kSelThreads + tid;
      uint32_t bin = 0xffffffffu;
      if (j < N_C) {
        const uint32_t key = keys[j];
        if ((key & pmask) == prefix) bin = (key >> shift) & 255u;
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (bin != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (tid < 32) {
      uint32_t loc[8], sum = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        loc[t] = hist[lane * 8 + t];
        sum += loc[t];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - sum;
      if (excl < k && k <= incl) {
        uint32_t c = excl;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (c + loc[t] >= k) {
            s_prefix = prefix | ((uint32_t)(lane * 8 + t) << shift);
            s_k = k - c;
            break;
          }
          c += loc[t];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    k = s_k;
    pmask |= 255u << shift;
  }
  const uint32_t T = prefix, k_eq = k;  // take all keys < T and the first k_eq keys == T

  // 3. slot-ordered listing: pos(j) = #(key < T before j) + min(#(key == T before j), k_eq).
  uint32_t less_base = 0, eq_base = 0;
  for (int r = 0; r < n_round; ++r) {
    const int j = r * kSelThreads + tid;
    uint32_t key = 0xffffffffu;
    bool valid = j < N_C;
    if (valid) key = keys[j];
    const uint32_t is_less = valid && key < T, is_eq = valid && key == T;
    const uint32_t ex = block_exclusive_scan((is_less << 16) | is_eq, warp_tot, &s_total);
    const uint32_t tot = s_total;
    const uint32_t less_before = less_base + (ex >> 16), eq_before = eq_base + (ex & 0xffffu);
    if (is_less || (is_eq && eq_before < k_eq)) {
      const uint32_t pos = less_before + min(eq_before, k_eq);
      list[pos] = j;
      if (sout) sout[pos] = j;
      tp[j] = P + (int)pos;
      sc[j] = 0.f;
    }
    less_base += tot >> 16;
    eq_base += tot & 0xffffu;
    __syncthreads();  // s_total is rewritten by the next round
  }
}

// ---- row quantizer ------------------------------------------------------------
// One warp per row of d bf16 values; lane handles element pairs lane, lane+32, ...
template <int KV>
__device__ __forceinline__ void quantize_row_warp(const __nv_bfloat16 *__restrict__ x, int d,
                                                  uint8_t *__restrict__ out, __half *scale_out) {
  constexpr int qmax = KV == H2OKV_I8 ? 127 : 7;
  const int lane = threadIdx.x & 31;
  const __nv_bfloat162 *x2 = reinterpret_cast<const __nv_bfloat162 *>(x);
  float amax = 0.f;
  for (int p = lane; p < d / 2; p += 32) {
    const float2 v = __bfloat1622float2(x2[p]);
    amax = fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  float r = amax / (float)qmax;  // IEEE division
  r = fminf(r, 65504.f);
  const __half hs = __float2half_rn(r);
  const float s = __half2float(hs);
  if (lane == 0) *scale_out = hs;
  for (int p = lane; p < d / 2; p += 32) {
    const float2 v = __bfloat1622float2(x2[p]);
    int qa = 0, qb = 0;
    if (s > 0.f) {
      qa = (int)fminf(fmaxf(rintf(v.x / s), (float)-qmax), (float)qmax);
      qb = (int)fminf(fmaxf(rintf(v.y / s), (float)-qmax), (float)qmax);
    }
    if (KV == H2OKV_I8) {
      out[2 * p] = (uint8_t)(int8_t)qa;
      out[2 * p + 1] = (uint8_t)(int8_t)qb;
    } else {
      out[p] = (uint8_t)((qa & 0xF) | ((qb & 0xF) << 4));
    }
  }
}

template <int KV>
__device__ __forceinline__ void copy_row_warp(const void *__restrict__ src, void *__restrict__ dst,
                                              int d) {
  const int lane = threadIdx.x & 31;
  const int words = KV == H2OKV_F32 ? d : d / 2;  // 32-bit words per row
  const uint32_t *s = reinterpret_cast<const uint32_t *>(src);
  uint32_t *o = reinterpret_cast<uint32_t *>(dst);
  for (int i = lane; i < words; i += 32) o[i] = s[i];
}

template <int KV>
__global__ void __launch_bounds__(256)
    scatter_kernel(const void *__restrict__ k_new, const void *__restrict__ v_new,
                   uint8_t *__restrict__ keys, uint8_t *__restrict__ values,
                   __half *__restrict__ k_scales, __half *__restrict__ v_scales,
                   const int32_t *__restrict__ slot_list, int n_rows, int S, int max_chunk,
                   int N_C, int d, size_t row_bytes, size_t in_row_bytes) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const int bh = row / S, k = row - bh * S;
  const int slot = slot_list[(size_t)bh * max_chunk + k];
  const size_t dst_row = (size_t)bh * N_C + slot;
  const uint8_t *ksrc = reinterpret_cast<const uint8_t *>(k_new) + (size_t)row * in_row_bytes;
  const uint8_t *vsrc = reinterpret_cast<const uint8_t *>(v_new) + (size_t)row * in_row_bytes;
  if constexpr (KV == H2OKV_I8 || KV == H2OKV_I4) {
    quantize_row_warp<KV>(reinterpret_cast<const __nv_bfloat16 *>(ksrc), d,
                          keys + dst_row * row_bytes, k_scales + dst_row);
    quantize_row_warp<KV>(reinterpret_cast<const __nv_bfloat16 *>(vsrc), d,
                          values + dst_row * row_bytes, v_scales + dst_row);
  } else {
    copy_row_warp<KV>(ksrc, keys + dst_row * row_bytes, d);
    copy_row_warp<KV>(vsrc, values + dst_row * row_bytes, d);
  }
}

template <int KV>
__global__ void __launch_bounds__(256)
    quantize_kernel(const __nv_bfloat16 *__restrict__ x, int64_t n_rows, int d,
                    uint8_t *__restrict__ codes, __half *__restrict__ scales, size_t row_bytes) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  quantize_row_warp<KV>(x + row * d, d, codes + row * row_bytes, scales + row);
}

__global__ void init_kernel(int32_t *__restrict__ token_pos, float *__restrict__ scores,
                            size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    token_pos[i] = kEmptyPos;
    scores[i] = 0.f;
  }
}

}  // namespace

int launch_init_cache(h2okv_cache *c, cudaStream_t st) {
  const size_t n = (size_t)c->desc.batch * c->desc.n_kv_heads * c->desc.capacity;
  if (cudaMemsetAsync(reinterpret_cast<uint8_t *>(c->bufs.workspace) + c->ws.status, 0, 4, st) !=
      cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaMemsetAsync(status) failed");
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  init_kernel<<<blocks, 256, 0, st>>>(c->bufs.token_pos, c->bufs.scores, n);
  return check_launch("init_kernel");
}

int launch_evict_insert(h2okv_cache *c, const float *w_prev, const void *k_new, const void *v_new,
                        int S, int64_t P, int32_t *slots_out, cudaStream_t st) {
  const h2okv_cache_desc &d = c->desc;
  const int BH = d.batch * d.n_kv_heads;
  const int mode = S == 0 ? 0 : (c->n_filled + S <= d.capacity ? 1 : 2);
  uint8_t *ws = reinterpret_cast<uint8_t *>(c->bufs.workspace);
  int32_t *slot_list = reinterpret_cast<int32_t *>(ws + c->ws.slot_list);
  uint32_t *gkeys = nullptr;
  size_t smem = 0;
  if (mode == 2) {
    if (d.capacity > kSmemKeyCap)
      gkeys = reinterpret_cast<uint32_t *>(ws + c->ws.sel_keys);
    else
      smem = (size_t)d.capacity * 4;
  }
  if (smem > 48 * 1024) {
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
      cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemKeyCap * 4);
      if (e != cudaSuccess)
        return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(select_kernel): %s",
                         cudaGetErrorString(e));
      configured_dev = dev;
    }
  }
  select_kernel<<<BH, kSelThreads, smem, st>>>(c->bufs.scores, w_prev, c->bufs.token_pos,
                                                d.capacity, S, (int)P, mode, c->n_filled,
                                                d.max_chunk, slot_list, slots_out, gkeys);
  int rc = check_launch("select_kernel");
  if (rc || S == 0) return rc;

  const int n_rows = BH * S;
  const int blocks = (n_rows + 7) / 8;
  const size_t in_row = (size_t)d.head_dim * (d.q_dtype == H2OKV_F32 ? 4 : 2);
  uint8_t *keys = reinterpret_cast<uint8_t *>(c->bufs.keys);
  uint8_t *vals = reinterpret_cast<uint8_t *>(c->bufs.values);
  __half *ks = reinterpret_cast<__half *>(c->bufs.k_scales);
  __half *vs = reinterpret_cast<__half *>(c->bufs.v_scales);
#define H2OKV_SCATTER(KV)                                                                   \
  scatter_kernel<KV><<<blocks, 256, 0, st>>>(k_new, v_new, keys, vals, ks, vs, slot_list,  \
                                             n_rows, S, d.max_chunk, d.capacity, d.head_dim, \
                                             c->row_bytes, in_row)
  switch (d.kv_dtype) {
    case H2OKV_F32: H2OKV_SCATTER(H2OKV_F32); break;
    case H2OKV_BF16: H2OKV_SCATTER(H2OKV_BF16); break;
    case H2OKV_I8: H2OKV_SCATTER(H2OKV_I8); break;
    case H2OKV_I4: H2OKV_SCATTER(H2OKV_I4); break;
  }
#undef H2OKV_SCATTER
  return check_launch("scatter_kernel");
}

int launch_quantize(int kv_dtype, const __nv_bfloat16 *x, int64_t n_rows, int d, void *codes,
                    __half *scales, cudaStream_t st) {
  const int64_t blocks = (n_rows + 7) / 8;
  if (blocks > INT32_MAX) return set_error(H2OKV_ERR_INVALID_ARG, "too many rows");
  const size_t rb = kv_row_bytes(kv_dtype, d);
  if (kv_dtype == H2OKV_I8)
    quantize_kernel<H2OKV_I8><<<(unsigned)blocks, 256, 0, st>>>(
        x, n_rows, d, reinterpret_cast<uint8_t *>(codes), scales, rb);
  else
    quantize_kernel<H2OKV_I4><<<(unsigned)blocks, 256, 0, st>>>(
        x, n_rows, d, reinterpret_cast<uint8_t *>(codes), scales, rb);
  return check_launch("quantize_kernel");
}

}  // namespace h2okv
