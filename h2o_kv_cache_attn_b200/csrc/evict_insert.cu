// H2O score update, lowest-score slot selection and overwrite of the chosen
// slots ("Learning how to Forget", §3.1 cache filled left to right then a
// per-(b, h) policy; §3.1.1 cumulative H2O score, lowest score evicted;
// §A.5.3 keys' = scatter(keys, index, key_new)), plus the 8/4-bit row
// quantizer used on insert.
//
// One launch per call: evict_kernel runs a thread-block cluster of CL CTAs per
// (b, h_k).  Each CTA holds a contiguous slice of the N_C slots in registers
// (IPT consecutive slots per thread) and
//   1. folds w_prev into the float32 scores and forms order-preserving uint32
//      selection keys (0 for an empty slot, so empty slots come first);
//   2. finds the S-th smallest key with a 4-pass, 8-bit radix select: each CTA
//      builds a 256-bin histogram of its slice, the cluster sums them through
//      distributed shared memory, every CTA picks the same bin;
//   3. lists the chosen slots in slot order (token k -> k-th smallest slot):
//      a block scan plus a cluster prefix of per-CTA counts gives each chosen
//      slot its position; the slot of position k is sent to CTA k % CL;
//   4. copies (or quantizes) the new key/value rows k = rank, rank + CL, ...
//      into their slots.
// While the cache is still filling (n_filled + S <= N_C) the slots are
// n_filled + k and steps 2-3 are skipped.  No scratch memory in global memory.
// The quantizer must agree bit for bit with an IEEE float32 reference: it uses
// correctly rounded division, rintf and __float2half_rn only (this file is
// never built with fast-math).
#include <cooperative_groups.h>

#include "h2okv_internal.cuh"

namespace h2okv {
namespace {

constexpr int kEvThreads = 256;   // threads per CTA of the eviction kernel
constexpr int kEvictCluster = 8;  // CTAs per (b, h_k): a portable cluster size
constexpr int kEvWarps = kEvThreads / 32;

// Unsigned key with the order of the float: -0 and +0 map to the same key;
// every non-NaN score maps to a key >= 1 so that 0 can mark an empty slot.
__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7fffffffu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of one uint32 per thread (blockDim.x == kEvThreads).
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
    uint32_t wv = lane < kEvWarps ? warp_tot[lane] : 0u;
    uint32_t wincl = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t t = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += t;
    }
    if (lane < kEvWarps) warp_tot[lane] = wincl - wv;
    if (lane == kEvWarps - 1) *total = wincl;
  }
  __syncthreads();
  return warp_tot[warp] + incl - v;
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

struct EvictArgs {
  float *scores;
  const float *w_prev;
  int32_t *token_pos;
  const uint8_t *k_new, *v_new;
  uint8_t *keys, *values;
  __half *k_scales, *v_scales;
  int32_t *slots_out;
  const int32_t *slots_in;  // replay: the slots to write (mode 3)
  uint8_t *dk, *dv;         // delta outputs (or null): overwritten rows [B][H_k][S][row bytes]
  __half *dks, *dvs;        //   their scales (quantized caches)
  int32_t *dpos;            //   their token positions [B][H_k][S]
  int *status;              // device status word (replayed slot outside the cache)
  int N_C, S, P, mode, n_filled, d, slice, score_mode, nbat, Hk;
  size_t row_bytes, in_row_bytes;
};

constexpr int kCopyUnroll = 8;   // 16-byte pieces per thread in flight in the row copy
constexpr int kQuantUnroll = 4;  // rows per lane segment in flight in the row quantizer

// The rows of one chunk row set: chunk rows k = rank + CL * m (m = 0 .. n_rows - 1) of
// (batch row, KV head) at cache offset gbase (slots) and chunk offset rbase (rows) go to
// slot slot_of(m) (negative: skipped).
struct RowSet {
  size_t gbase, rbase;
};

// f32 / bf16 caches: the key and value rows are cut into 16-byte pieces spread over the
// whole CTA (consecutive threads take consecutive pieces of a row), and every thread loads
// kCopyUnroll pieces before it stores any, so a launch waits on memory a few times in all
// rather than once per row.  With delta outputs the same thread first reads the piece it
// overwrites.
template <bool FULL, typename SlotOf>
__device__ __forceinline__ void copy_rows_cta(const EvictArgs &a, RowSet rs, int rank, int CL,
                                              int n_rows, SlotOf slot_of) {
  const int C = (int)(a.row_bytes / 16);  // 16-byte pieces per row (row_bytes % 16 == 0)
  const int total = n_rows * 2 * C;
  const bool dl = FULL && a.dk != nullptr;
  for (int base = threadIdx.x; base < total; base += kEvThreads * kCopyUnroll) {
    uint4 r[kCopyUnroll], old[kCopyUnroll];
    uint4 *dst[kCopyUnroll];
    uint4 *ddst[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const int e = base + u * kEvThreads;
      dst[u] = nullptr;
      ddst[u] = nullptr;
      if (e < total) {
        const int c = e % C, rest = e / C, t = rest & 1, m = rest >> 1;
        const size_t row = rs.rbase + rank + (size_t)CL * m;
        const uint8_t *src = (t ? a.v_new : a.k_new) + row * a.in_row_bytes;
        r[u] = __ldcs(reinterpret_cast<const uint4 *>(src) + c);
        const int slot = slot_of(m);
        if (slot >= 0) {
          dst[u] = reinterpret_cast<uint4 *>((t ? a.values : a.keys) +
                                             (rs.gbase + (size_t)slot) * a.row_bytes) + c;
          if (dl) {
            old[u] = *dst[u];
            ddst[u] = reinterpret_cast<uint4 *>((t ? a.dv : a.dk) + row * a.row_bytes) + c;
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      if (ddst[u]) *ddst[u] = old[u];
      if (dst[u]) *dst[u] = r[u];
    }
  }
}

// int8 / int4 caches: one row per segment of L lanes (L = the smallest power of two
// >= d / 8); lane i of a segment holds elements 8i .. 8i + 7 of the row.  A warp covers
// 32 / L rows per pass and keeps kQuantUnroll passes in flight.  Per row, the same
// arithmetic as the per-row quantizer: absmax, IEEE division by qmax, clamp to the fp16
// range, round to fp16, then rint(x / scale) clamped to [-qmax, qmax].  With delta
// outputs each lane first copies the codes (and lane 0 the scale) it overwrites.
template <int KV, bool FULL, typename SlotOf>
__device__ __forceinline__ void quantize_rows_cta(const EvictArgs &a, RowSet rs, int rank, int CL,
                                                  int n_rows, SlotOf slot_of) {
  constexpr int qmax = KV == H2OKV_I8 ? 127 : 7;
  const int G = a.d / 8;
  int L = 1;
  while (L < G) L <<= 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = lane / L, li = lane % L, segs = 32 / L;
  const int items = n_rows * 2;  // (m, t): t = 0 key row, 1 value row
  const bool dl = FULL && a.dk != nullptr;
  for (int p0 = 0; (p0 * kEvWarps + warp) * segs < items; p0 += kQuantUnroll) {
    uint4 x[kQuantUnroll];
    bool ok[kQuantUnroll];
    int slot[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int item = ((p0 + u) * kEvWarps + warp) * segs + seg;
      ok[u] = item < items && li < G;
      x[u] = make_uint4(0u, 0u, 0u, 0u);
      slot[u] = -1;
      if (ok[u]) {
        const int t = item & 1, m = item >> 1;
        slot[u] = slot_of(m);
        const size_t row = rs.rbase + rank + (size_t)CL * m;
        const uint8_t *src = (t ? a.v_new : a.k_new) + row * a.in_row_bytes;
        x[u] = __ldcs(reinterpret_cast<const uint4 *>(src) + li);
      }
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      float v[8];
      const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&x[u]);
      float amax = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(h2[q]);
        v[2 * q] = f.x;
        v[2 * q + 1] = f.y;
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
      for (int o = L >> 1; o > 0; o >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      float r = amax / (float)qmax;  // IEEE division
      r = fminf(r, 65504.f);
      const __half hs = __float2half_rn(r);
      const float s = __half2float(hs);
      int qc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        qc[q] = s > 0.f ? (int)fminf(fmaxf(rintf(v[q] / s), (float)-qmax), (float)qmax) : 0;
      if (!ok[u] || slot[u] < 0) continue;
      const int item = ((p0 + u) * kEvWarps + warp) * segs + seg;
      const int t = item & 1, m = item >> 1;
      const size_t drow = rs.gbase + (size_t)slot[u];
      const size_t crow = rs.rbase + rank + (size_t)CL * m;
      uint8_t *codes = (t ? a.values : a.keys) + drow * a.row_bytes;
      __half *sdst = (t ? a.v_scales : a.k_scales) + drow;
      if (dl) {
        uint8_t *dcodes = (t ? a.dv : a.dk) + crow * a.row_bytes;
        if (li == 0) (t ? a.dvs : a.dks)[crow] = *sdst;
        if (KV == H2OKV_I8)
          reinterpret_cast<uint2 *>(dcodes)[li] = reinterpret_cast<const uint2 *>(codes)[li];
        else
          reinterpret_cast<uint32_t *>(dcodes)[li] = reinterpret_cast<const uint32_t *>(codes)[li];
      }
      if (li == 0) *sdst = hs;
      if (KV == H2OKV_I8) {
        uint32_t lo = 0u, hi = 0u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          lo |= ((uint32_t)(qc[q] & 0xFF)) << (8 * q);
          hi |= ((uint32_t)(qc[q + 4] & 0xFF)) << (8 * q);
        }
        reinterpret_cast<uint2 *>(codes)[li] = make_uint2(lo, hi);
      } else {
        uint32_t w = 0u;  // element 2i in the low nibble of byte i
#pragma unroll
        for (int q = 0; q < 8; ++q) w |= ((uint32_t)(qc[q] & 0xF)) << (4 * q);
        reinterpret_cast<uint32_t *>(codes)[li] = w;
      }
    }
  }
}

template <int KV, bool FULL, typename SlotOf>
__device__ __forceinline__ void insert_rows_cta(const EvictArgs &a, RowSet rs, int rank, int CL,
                                                SlotOf slot_of) {
  const int n_rows = rank < a.S ? (a.S - rank + CL - 1) / CL : 0;
  if constexpr (KV == H2OKV_I8 || KV == H2OKV_I4)
    quantize_rows_cta<KV, FULL>(a, rs, rank, CL, n_rows, slot_of);
  else
    copy_rows_cta<FULL>(a, rs, rank, CL, n_rows, slot_of);
}

template <int IPT>
__device__ __forceinline__ void store_slice(float *dst, const float (&v)[IPT],
                                            const bool (&valid)[IPT], bool vec) {
  if constexpr (IPT % 4 == 0) {
    if (vec) {
#pragma unroll
      for (int i = 0; i < IPT; i += 4)
        *reinterpret_cast<float4 *>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      return;
    }
  }
  {
#pragma unroll
    for (int i = 0; i < IPT; ++i)
      if (valid[i]) dst[i] = v[i];
  }
}

// Slot j of a chunk row set receives chunk row k: bookkeeping of the slot (old token
// position to the delta output, new token position, score 0 unless the caller stores
// the slice's scores afterwards, slot list).
template <bool FULL>
__device__ __forceinline__ void claim_slot(const EvictArgs &a, RowSet rs, int j, int k,
                                           bool zero_score = true) {
  const size_t gs = rs.gbase + (size_t)j, rk = rs.rbase + (size_t)k;
  if (FULL && a.dpos) a.dpos[rk] = a.token_pos[gs];
  a.token_pos[gs] = a.P + k;
  if (zero_score) a.scores[gs] = 0.f;
  if (a.slots_out) a.slots_out[rk] = j;
}

// mode 0: fold w_prev only (S = 0); 1: fill slots n_filled.. (no occupied slot is
// touched); 2: generic choice (empty slots first, then lowest selection keys);
// 3: replay (write the given slots).  One cluster per (batch row, KV head), or per KV
// head for all batch rows together (score variant h2o_orig: nbat > 1).
// FULL: the general kernel (h2o_orig over several batch rows, replay, delta outputs); the
// other instance is the plain per-(b, h_k) choice, built without those paths.
template <int KV, int IPT, bool FULL>
__global__ void __launch_bounds__(kEvThreads) evict_kernel(const EvictArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int gi = blockIdx.x / CL;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nb = FULL ? a.nbat : 1;
  const int b_first = nb > 1 ? 0 : gi / a.Hk, h = nb > 1 ? gi : gi % a.Hk;
  auto rows_of = [&](int bb) {
    const size_t bh = (size_t)(b_first + bb) * a.Hk + h;
    return RowSet{bh * (size_t)a.N_C, bh * (size_t)a.S};
  };

  __shared__ uint32_t hist[2][256];
  __shared__ uint32_t tot_bins[256];
  __shared__ uint32_t warp_tot[kEvWarps];
  __shared__ uint32_t s_prefix, s_k, s_total;
  __shared__ uint32_t cta_less, cta_eq;
  extern __shared__ int32_t rowslot[];  // [ceil(S / CL)]: slot of chunk row rank + CL * m

  const int j0 = rank * a.slice + tid * IPT;
  float sc[IPT], ksum[IPT];
  int32_t tp[IPT];
  uint32_t key[IPT];
  bool valid[IPT];
#pragma unroll
  for (int i = 0; i < IPT; ++i) {
    valid[i] = j0 + i < a.N_C;
    tp[i] = kEmptyPos;
    ksum[i] = 0.f;
  }
  // one batch row choosing for itself: its folded scores are stored once, after the
  // choice, with the chosen slots at 0 (the stores then overlap nothing else)
  const bool defer_store = a.mode == 2 && nb == 1;
  bool vec0 = false;
  // ---- fold w_prev into the scores of every batch row of this set ----------------
  for (int bb = 0; bb < nb; ++bb) {
    const size_t gbase = rows_of(bb).gbase;
    float wp[IPT];
#pragma unroll
    for (int i = 0; i < IPT; ++i) {
      sc[i] = 0.f;
      wp[i] = 0.f;
    }
    const bool want_tp = bb == 0 && a.mode == 2;
    // 16-byte loads when this thread's slots are whole and aligned, else one by one
    const bool vec = IPT % 4 == 0 && j0 + IPT <= a.N_C &&
                     ((reinterpret_cast<uintptr_t>(a.scores + gbase + j0) |
                       reinterpret_cast<uintptr_t>(a.token_pos + gbase + j0) |
                       (a.w_prev ? reinterpret_cast<uintptr_t>(a.w_prev + gbase + j0) : 0u)) &
                      15u) == 0u;
    bool loaded = false;
    if constexpr (IPT % 4 == 0) {
      if (vec) {
#pragma unroll
        for (int i = 0; i < IPT; i += 4) {
          *reinterpret_cast<float4 *>(&sc[i]) =
              *reinterpret_cast<const float4 *>(a.scores + gbase + j0 + i);
          if (a.w_prev)
            *reinterpret_cast<float4 *>(&wp[i]) =
                __ldcs(reinterpret_cast<const float4 *>(a.w_prev + gbase + j0 + i));
          if (want_tp)
            *reinterpret_cast<int4 *>(&tp[i]) =
                *reinterpret_cast<const int4 *>(a.token_pos + gbase + j0 + i);
        }
        loaded = true;
      }
    }
    if (!loaded) {
#pragma unroll
      for (int i = 0; i < IPT; ++i) {
        if (!valid[i]) continue;
        sc[i] = a.scores[gbase + j0 + i];
        if (a.w_prev) wp[i] = a.w_prev[gbase + j0 + i];
        if (want_tp) tp[i] = a.token_pos[gbase + j0 + i];
      }
    }
#pragma unroll
    for (int i = 0; i < IPT; ++i) {
      if (a.w_prev) sc[i] = __fadd_rn(sc[i], wp[i]);
      ksum[i] = bb == 0 ? sc[i] : __fadd_rn(ksum[i], sc[i]);  // h2o_orig: batch order
    }
    if (a.w_prev && !defer_store) store_slice<IPT>(a.scores + gbase + j0, sc, valid, vec);
    if (bb == 0) vec0 = vec;
  }

  if (a.mode == 1) {
    // while filling: chunk row k takes slot n_filled + k (same slot for every batch row)
#pragma unroll
    for (int i = 0; i < IPT; ++i) {
      const int k = j0 + i - a.n_filled;
      if (valid[i] && k >= 0 && k < a.S)
        for (int bb = 0; bb < nb; ++bb) claim_slot<FULL>(a, rows_of(bb), j0 + i, k);
    }
    const int first = a.n_filled + rank;
    for (int bb = 0; bb < nb; ++bb)
      insert_rows_cta<KV, FULL>(a, rows_of(bb), rank, CL, [&](int m) { return first + CL * m; });
    return;
  }
  if (FULL && a.mode == 3) {
    // replay: every fold store of the cluster lands before a replayed slot is reset
    cluster.sync();
    for (int bb = 0; bb < nb; ++bb) {
      const RowSet rs = rows_of(bb);
      auto slot_of = [&](int m) -> int {
        const int j = a.slots_in[rs.rbase + rank + (size_t)CL * m];
        return (j >= 0 && j < a.N_C) ? j : -1;
      };
      for (int m = tid; rank + CL * m < a.S; m += kEvThreads) {
        const int j = slot_of(m);
        if (j < 0)
          atomicExch(a.status, H2OKV_ERR_INVALID_ARG);
        else
          claim_slot<FULL>(a, rs, j, rank + CL * m);
      }
      insert_rows_cta<KV, FULL>(a, rs, rank, CL, slot_of);
    }
    return;
  }
  if (a.mode != 2) return;

  // ---- selection keys ----------------------------------------------------------------
#pragma unroll
  for (int i = 0; i < IPT; ++i) {
    float kv = ksum[i];
    if (a.score_mode == 1) {  // h2o_norm: score / (P - t(b, h, j)), age at least 1
      const int age = max(a.P - tp[i], 1);
      kv = __fdiv_rn(kv, (float)age);
    }
    key[i] = (valid[i] && tp[i] != kEmptyPos) ? order_key(kv) : 0u;
  }

  // ---- radix select of the S-th smallest key over the whole cluster --------------
  uint32_t prefix = 0u, pmask = 0u, kk = (uint32_t)a.S;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t *h = hist[pass & 1];
    h[tid] = 0u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < IPT; ++i) {
      const uint32_t bin =
          (valid[i] && (key[i] & pmask) == prefix) ? (key[i] >> shift) & 255u : 0xffffffffu;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (bin != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&h[bin], __popc(peers));
    }
    cluster.sync();  // every CTA's histogram of this pass is complete
    uint32_t sum = 0u;
    for (int q = 0; q < CL; ++q) sum += cluster.map_shared_rank(h, q)[tid];
    tot_bins[tid] = sum;
    __syncthreads();
    if (warp == 0) {
      uint32_t loc[8], lsum = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        loc[t] = tot_bins[lane * 8 + t];
        lsum += loc[t];
      }
      uint32_t incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - lsum;
      if (excl < kk && kk <= incl) {
        uint32_t c = excl;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (c + loc[t] >= kk) {
            s_prefix = prefix | ((uint32_t)(lane * 8 + t) << shift);
            s_k = kk - c;
            break;
          }
          c += loc[t];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    kk = s_k;
    pmask |= 255u << shift;
  }
  const uint32_t T = prefix, k_eq = kk;  // take every key < T and the first k_eq keys == T

  // ---- chosen slots in slot order ---------------------------------------------------
  uint32_t nl = 0, ne = 0;
#pragma unroll
  for (int i = 0; i < IPT; ++i) {
    nl += (valid[i] && key[i] < T) ? 1u : 0u;
    ne += (valid[i] && key[i] == T) ? 1u : 0u;
  }
  // per-thread counts <= IPT and per-CTA totals <= kEvThreads * IPT < 65536: pack 16 + 16 bits
  const uint32_t ex = block_exclusive_scan((nl << 16) | ne, warp_tot, &s_total);
  if (tid == 0) {
    cta_less = s_total >> 16;
    cta_eq = s_total & 0xffffu;
  }
  cluster.sync();  // per-CTA totals visible to the cluster
  uint32_t base_less = 0, base_eq = 0;
  for (int q = 0; q < rank; ++q) {
    base_less += *cluster.map_shared_rank(&cta_less, q);
    base_eq += *cluster.map_shared_rank(&cta_eq, q);
  }
  uint32_t less_before = base_less + (ex >> 16), eq_before = base_eq + (ex & 0xffffu);
#pragma unroll
  for (int i = 0; i < IPT; ++i) {
    if (!valid[i]) continue;
    const int j = j0 + i;
    bool take = false;
    uint32_t pos = 0;
    if (key[i] < T) {
      take = true;
      pos = less_before + min(eq_before, k_eq);
      ++less_before;
    } else if (key[i] == T) {
      take = eq_before < k_eq;
      pos = less_before + eq_before;
      ++eq_before;
    }
    if (take) {
      if (defer_store) sc[i] = 0.f;
      for (int bb = 0; bb < nb; ++bb) claim_slot<FULL>(a, rows_of(bb), j, (int)pos, !defer_store);
      int32_t *dst = cluster.map_shared_rank(rowslot, (int)(pos % (uint32_t)CL));
      dst[pos / (uint32_t)CL] = j;
    }
  }
  if (defer_store) store_slice<IPT>(a.scores + rows_of(0).gbase + j0, sc, valid, vec0);
  cluster.sync();  // rowslot lists complete

  // ---- insert the chunk's rows k = rank, rank + CL, ... -----------------------------
  for (int bb = 0; bb < nb; ++bb)
    insert_rows_cta<KV, FULL>(a, rows_of(bb), rank, CL, [&](int m) { return rowslot[m]; });
}

template <int KV>
__global__ void __launch_bounds__(256)
    quantize_kernel(const __nv_bfloat16 *__restrict__ x, int64_t n_rows, int d,
                    uint8_t *__restrict__ codes, __half *__restrict__ scales, size_t row_bytes) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  quantize_row_warp<KV>(x + row * d, d, codes + row * row_bytes, scales + row);
}

// Delta rows back into their slots (one warp per chunk row; 4-byte words).
__global__ void __launch_bounds__(256)
    restore_kernel(const int32_t *__restrict__ slots, int64_t n_rows, int S, int N_C,
                   size_t row_bytes, const uint8_t *__restrict__ dk, const uint8_t *__restrict__ dv,
                   const __half *__restrict__ dks, const __half *__restrict__ dvs,
                   const int32_t *__restrict__ dpos, uint8_t *keys, uint8_t *values,
                   __half *k_scales, __half *v_scales, int32_t *token_pos, int *status) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const int j = slots[row];
  if (j < 0 || j >= N_C) {
    if (lane == 0) atomicExch(status, H2OKV_ERR_INVALID_ARG);
    return;
  }
  const size_t dst = (size_t)(row / S) * N_C + j;  // slot j of this row's (b, h_k)
  const int words = (int)(row_bytes / 4);
  const uint32_t *sk = reinterpret_cast<const uint32_t *>(dk + row * row_bytes);
  const uint32_t *sv = reinterpret_cast<const uint32_t *>(dv + row * row_bytes);
  uint32_t *tk = reinterpret_cast<uint32_t *>(keys + dst * row_bytes);
  uint32_t *tv = reinterpret_cast<uint32_t *>(values + dst * row_bytes);
  for (int w = lane; w < words; w += 32) {
    tk[w] = sk[w];
    tv[w] = sv[w];
  }
  if (lane == 0) {
    if (k_scales && dks) k_scales[dst] = dks[row];
    if (v_scales && dvs) v_scales[dst] = dvs[row];
    token_pos[dst] = dpos[row];
  }
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

template <int KV, int IPT, bool FULL>
static int launch_evict_t(const EvictArgs &a, int n_groups, int CL, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(n_groups * CL));
  cfg.blockDim = dim3(kEvThreads);
  cfg.dynamicSmemBytes = (size_t)((a.S + CL - 1) / CL) * 4;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cfg.dynamicSmemBytes > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(evict_kernel<KV, IPT, FULL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)cfg.dynamicSmemBytes);
    if (e != cudaSuccess)
      return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(evict_kernel): %s",
                       cudaGetErrorString(e));
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, evict_kernel<KV, IPT, FULL>, a);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "evict_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("evict_kernel");
}

template <int KV, bool FULL>
static int launch_evict_kv(const EvictArgs &a, int n_groups, int CL, int ipt, cudaStream_t st) {
  switch (ipt) {
    case 1: return launch_evict_t<KV, 1, FULL>(a, n_groups, CL, st);
    case 2: return launch_evict_t<KV, 2, FULL>(a, n_groups, CL, st);
    case 4: return launch_evict_t<KV, 4, FULL>(a, n_groups, CL, st);
    case 8: return launch_evict_t<KV, 8, FULL>(a, n_groups, CL, st);
    case 16: return launch_evict_t<KV, 16, FULL>(a, n_groups, CL, st);
    case 32: return launch_evict_t<KV, 32, FULL>(a, n_groups, CL, st);
  }
  return set_error(H2OKV_ERR_UNSUPPORTED, "capacity too large for the eviction kernel");
}

int launch_evict_insert(h2okv_cache *c, const float *w_prev, const void *k_new, const void *v_new,
                        int S, int64_t P, int32_t *slots_out, const int32_t *slots_in,
                        const h2okv_delta *delta, cudaStream_t st) {
  const h2okv_cache_desc &d = c->desc;
  EvictArgs a;
  a.scores = c->bufs.scores;
  a.w_prev = w_prev;
  a.token_pos = c->bufs.token_pos;
  a.k_new = reinterpret_cast<const uint8_t *>(k_new);
  a.v_new = reinterpret_cast<const uint8_t *>(v_new);
  a.keys = reinterpret_cast<uint8_t *>(c->bufs.keys);
  a.values = reinterpret_cast<uint8_t *>(c->bufs.values);
  a.k_scales = reinterpret_cast<__half *>(c->bufs.k_scales);
  a.v_scales = reinterpret_cast<__half *>(c->bufs.v_scales);
  a.slots_out = slots_out;
  a.slots_in = slots_in;
  a.dk = delta ? reinterpret_cast<uint8_t *>(delta->keys) : nullptr;
  a.dv = delta ? reinterpret_cast<uint8_t *>(delta->values) : nullptr;
  a.dks = delta ? reinterpret_cast<__half *>(delta->k_scales) : nullptr;
  a.dvs = delta ? reinterpret_cast<__half *>(delta->v_scales) : nullptr;
  a.dpos = delta ? delta->token_pos : nullptr;
  a.status = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(c->bufs.workspace) + c->ws.status);
  a.N_C = d.capacity;
  a.S = S;
  a.P = (int)P;
  a.mode = S == 0 ? 0 : (slots_in ? 3 : (c->n_filled + S <= d.capacity ? 1 : 2));
  a.score_mode = c->score_mode;
  a.Hk = d.n_kv_heads;
  // h2o_orig: one cluster per KV head selects for every batch row
  const bool orig = c->score_mode == H2OKV_SCORE_H2O_ORIG && a.mode == 2;
  a.nbat = orig ? d.batch : 1;
  a.n_filled = c->n_filled;
  a.d = d.head_dim;
  a.row_bytes = c->row_bytes;
  a.in_row_bytes = (size_t)d.head_dim * (d.q_dtype == H2OKV_F32 ? 4 : 2);
  // cluster size and slots per thread: CL * kEvThreads * IPT >= N_C
  const int CL = kEvictCluster;
  int ipt = 1;
  while ((int64_t)CL * kEvThreads * ipt < d.capacity) ipt *= 2;
  a.slice = kEvThreads * ipt;
  const int n_groups = orig ? d.n_kv_heads : d.batch * d.n_kv_heads;
  const bool full = orig || delta != nullptr || a.mode == 3;
  switch (d.kv_dtype) {
    case H2OKV_F32:
      return full ? launch_evict_kv<H2OKV_F32, true>(a, n_groups, CL, ipt, st)
                  : launch_evict_kv<H2OKV_F32, false>(a, n_groups, CL, ipt, st);
    case H2OKV_BF16:
      return full ? launch_evict_kv<H2OKV_BF16, true>(a, n_groups, CL, ipt, st)
                  : launch_evict_kv<H2OKV_BF16, false>(a, n_groups, CL, ipt, st);
    case H2OKV_I8:
      return full ? launch_evict_kv<H2OKV_I8, true>(a, n_groups, CL, ipt, st)
                  : launch_evict_kv<H2OKV_I8, false>(a, n_groups, CL, ipt, st);
    case H2OKV_I4:
      return full ? launch_evict_kv<H2OKV_I4, true>(a, n_groups, CL, ipt, st)
                  : launch_evict_kv<H2OKV_I4, false>(a, n_groups, CL, ipt, st);
  }
  return set_error(H2OKV_ERR_UNSUPPORTED, "kv dtype");
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

int launch_restore(h2okv_cache *c, const int32_t *slots, int S, const h2okv_delta *delta,
                   cudaStream_t st) {
  const h2okv_cache_desc &d = c->desc;
  const int64_t n_rows = (int64_t)d.batch * d.n_kv_heads * S;
  if (n_rows == 0) return H2OKV_OK;
  const bool quant = d.kv_dtype == H2OKV_I8 || d.kv_dtype == H2OKV_I4;
  restore_kernel<<<(unsigned)((n_rows + 7) / 8), 256, 0, st>>>(
      slots, n_rows, S, d.capacity, c->row_bytes, reinterpret_cast<const uint8_t *>(delta->keys),
      reinterpret_cast<const uint8_t *>(delta->values),
      quant ? reinterpret_cast<const __half *>(delta->k_scales) : nullptr,
      quant ? reinterpret_cast<const __half *>(delta->v_scales) : nullptr, delta->token_pos,
      reinterpret_cast<uint8_t *>(c->bufs.keys), reinterpret_cast<uint8_t *>(c->bufs.values),
      reinterpret_cast<__half *>(c->bufs.k_scales), reinterpret_cast<__half *>(c->bufs.v_scales),
      c->bufs.token_pos,
      reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(c->bufs.workspace) + c->ws.status));
  return check_launch("restore_kernel");
}

}  // namespace h2okv
