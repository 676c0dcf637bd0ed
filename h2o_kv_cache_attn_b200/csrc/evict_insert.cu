// H2O score update, lowest-score slot selection and overwrite of the chosen
// slots ("Learning how to Forget", §3.1 cache filled left to right then a
// per-(b, h) policy; §3.1.1 cumulative H2O score, lowest score evicted;
// §A.5.3 keys' = scatter(keys, index, key_new)), plus the 8/4-bit row
// quantizer used on insert.
//
// One call = up to three launches on the caller's stream, chained by programmatic
// dependent launch (each next kernel is scheduled early and waits for the previous
// one with griddepcontrol.wait):
//
//   evict_fold_kernel    C CTAs per group (a group is one (batch row, KV head), or one
//     KV head over every batch row for the h2o_orig variant), each over a slice of
//     the N_C slots: folds w_prev into the float32 scores and stores them; while the
//     cache is filling (n_filled + S <= N_C) it claims slots n_filled + k for the
//     chunk rows k; when choosing, it adds the slice's histogram of the top 11 bits
//     of the order-preserving selection keys (0 for an empty slot, so empty slots
//     come first) into the group's histogram in the workspace.
//   evict_choose_kernel  (choosing only) one CTA per group: finds the bin of the
//     S-th smallest key, marks the slots below it and in it (the candidates) in two
//     bitmasks, refines the threshold over the candidates (bits 20..10, 9..0; ties
//     go to the lowest slots) and lists the chosen slots in slot order.
//   evict_rows_kernel    over every chunk row, key and value: loads the new rows
//     while the earlier kernels run, then writes (copies, or quantizes for 8/4-bit
//     caches) each into its slot, saving the overwritten row first for the delta
//     encoding, and claims chosen or replayed slots (token position, score 0).
//
// A call over many caches of the same shape (independent layers) runs as the
// same three launches over every (cache, group), up to 48 caches per launch.  The
// quantizer must agree bit for bit with an IEEE float32 reference: it uses correctly
// rounded division and reciprocal, Markstein's correctly rounded quotient (quant_code)
// and __float2half_rn only (this file is never built with fast-math).
#include <mutex>

#include "h2okv_internal.cuh"
#include "tc_ptx.cuh"

namespace h2okv {
namespace {
using namespace ptx;

constexpr int kSelThreads = 512;  // threads of a select CTA
constexpr int kTopBits = 11;  // bits of the first histogram (key bits 31..21)
constexpr int kHistBins = 1 << kTopBits;
constexpr int kMidBins = 2048;  // key bits 20..10
constexpr int kLowBins = 1024;  // key bits 9..0
constexpr int kSmemKeysMax = 32768;  // largest N_C whose keys the last CTA keeps in shared memory
constexpr int kRowThreads = 256;     // threads of a row CTA
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kCopyUnroll = 8;   // 16-byte pieces per thread in flight in the row copy
constexpr int kQuantUnroll = 2;  // rows per lane segment in flight in the row quantizer
constexpr int kQuantChunks = 4;  // 8-element chunks of a row per lane (up to)

// ---- quantizer arithmetic ------------------------------------------------------------
// code = clamp(rint(x / s), -qmax, qmax) with x / s the correctly rounded float32
// quotient, without a division per element: Markstein's division (P. Markstein, IBM J.
// Res. Dev. 34(1), 1990): with y = RN(1/s) (one per row), q0 = RN(x y) is within one ulp
// of x / s, r = x - s q0 is exact (one FMA), and RN(q0 + r y) is RN(x / s).  The
// quotient is clamped first (which commutes with rounding to an integer for integer
// bounds), then rounded to nearest-even by adding and removing 1.5 * 2^23 (exact for
// |q| < 2^22).  For s > 0 only (scale 0 gives codes 0).
__device__ __forceinline__ int quant_code(float x, float s, float y, float qmax) {
  const float q0 = __fmul_rn(x, y);
  const float r = __fmaf_rn(-q0, s, x);
  float q = __fmaf_rn(r, y, q0);
  q = fminf(fmaxf(q, -qmax), qmax);
  return __float_as_int(__fadd_rn(q, 12582912.f)) - 0x4B400000;
}

// The same for two elements with packed float32 arithmetic (each lane of an f32x2
// operation is the IEEE float32 operation above); returns the bits of q + 1.5 * 2^23,
// whose low byte (low nibble) is the int8 (int4) code in two's complement.
__device__ __forceinline__ uint2 quant_bits2(float2 x, float s, float y, float qmax) {
  const float2 q0 = mul2(x, make_float2(y, y));
  const float2 r = fma2(q0, make_float2(-s, -s), x);
  float2 q = fma2(r, make_float2(y, y), q0);
  q.x = fminf(fmaxf(q.x, -qmax), qmax);
  q.y = fminf(fmaxf(q.y, -qmax), qmax);
  const float2 t = add2(q, make_float2(12582912.f, 12582912.f));
  return make_uint2(__float_as_uint(t.x), __float_as_uint(t.y));
}

// Unsigned key with the order of the float: -0 and +0 map to the same key;
// every non-NaN score maps to a key >= 1 so that 0 can mark an empty slot.
__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7fffffffu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// One cache of a call: its buffers, the caller's chunk buffers and its workspace.
struct EvTarget {
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
  uint32_t *hist;           // workspace: [groups][kHistBins] top-bit histograms, zero between calls
  uint32_t *arrive;         // workspace: [groups] arrival counters, zero between calls
  int32_t *slotlist;        // workspace: [groups][S] chosen slots in slot order (mode 2)
  int *status;              // device status word (replayed slot outside the cache)
};

template <int NT>
struct EvParams {
  EvTarget t[NT];
  int n_targets;
  int G;            // groups per cache: B * H_k, or H_k (h2o_orig: every batch row together)
  int nb;           // batch rows per group (1, or B for h2o_orig)
  int Hk, N_C, S, P, n_filled, d;
  int mode;         // 0 fold only (S = 0), 1 fill, 2 choose, 3 replay
  int score_mode;   // h2okv_score_mode
  int need_tp;      // the selection keys read token positions (empty slots, h2o_norm)
  int vec;          // N_C % 4 == 0: 16-byte loads and stores of score / position vectors
  int C;            // select CTAs per group
  int slice;        // slots per select CTA (a multiple of 4)
  int row_bytes, in_row_bytes;
  uint64_t wait_ns;  // limit of the choose kernel's wait on its bulk copies
};

template <int NT>
__device__ __forceinline__ size_t bh_of(const EvParams<NT> &p, int g, int bb) {
  return p.nb > 1 ? (size_t)bb * p.Hk + g : (size_t)g;
}

// ---- vector helpers: 4 consecutive slots j4 .. j4+3 below `end` ------------------
__device__ __forceinline__ void ld4(const float *base, int j4, int end, bool vec, float (&v)[4]) {
  if (vec && j4 + 4 <= end) {
    const float4 x = *reinterpret_cast<const float4 *>(base + j4);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = j4 + e < end ? base[j4 + e] : 0.f;
  }
}
__device__ __forceinline__ void ld4_cs(const float *base, int j4, int end, bool vec, float (&v)[4]) {
  if (vec && j4 + 4 <= end) {
    const float4 x = __ldcs(reinterpret_cast<const float4 *>(base + j4));
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = j4 + e < end ? __ldcs(base + j4 + e) : 0.f;
  }
}
__device__ __forceinline__ void ld4i(const int32_t *base, int j4, int end, bool vec,
                                     int32_t (&v)[4]) {
  if (vec && j4 + 4 <= end) {
    const int4 x = *reinterpret_cast<const int4 *>(base + j4);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = j4 + e < end ? base[j4 + e] : kEmptyPos;
  }
}
__device__ __forceinline__ void st4(float *base, int j4, int end, bool vec, const float (&v)[4]) {
  if (vec && j4 + 4 <= end) {
    *reinterpret_cast<float4 *>(base + j4) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (j4 + e < end) base[j4 + e] = v[e];
  }
}

// Shared-memory accesses by 32-bit shared addresses (explicit ld/st.shared).
__device__ __forceinline__ int lds32(uint32_t a) {
  int v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts32(uint32_t a, int v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// hs[bin] += 1 for the calling lane: lanes (of those active together) that share a bin
// add once, with their count.  Selection keys are often crowded into a few bins (scores
// of one chunk's age are alike), where lane-by-lane atomics would serialize.
__device__ __forceinline__ void hist_add(uint32_t *hs, uint32_t bin) {
  const uint32_t peers = __match_any_sync(__activemask(), bin);
  if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hs[bin], __popc(peers));
}

// Selection key of one slot from its (folded) score sum over the group's batch rows and
// the token position of batch row 0.
__device__ __forceinline__ uint32_t sel_key(float ksum, int32_t tp, int score_mode, int P) {
  if (tp == kEmptyPos) return 0u;
  if (score_mode == H2OKV_SCORE_H2O_NORM) {  // score / (P - t(b, h, j)), age at least 1
    const int age = max(P - tp, 1);
    ksum = __fdiv_rn(ksum, (float)age);
  }
  return order_key(ksum);
}

// Block-wide exclusive scan over NTHR threads (warp_tot: NTHR / 32 entries).
template <int NTHR, typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T *warp_tot) {
  constexpr int kW = NTHR / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const T wv = lane < kW ? warp_tot[lane] : (T)0;
    T wincl = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const T t = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += t;
    }
    if (lane < kW) warp_tot[lane] = wincl - wv;
  }
  __syncthreads();
  const T r = warp_tot[warp] + incl - v;
  __syncthreads();  // warp_tot may be reused right away
  return r;
}

// The bin of hs[0 .. NBINS) that holds the kk-th smallest counted key (1-based): writes
// res[0] = bin, res[1] = kk minus the keys in lower bins.
template <int NTHR, int NBINS>
__device__ __forceinline__ void find_bin(const uint32_t *hs, uint32_t kk, uint32_t *warp_tot,
                                         uint32_t *res) {
  constexpr int per = NBINS / NTHR;
  const int t = threadIdx.x;
  uint32_t loc = 0;
#pragma unroll
  for (int i = 0; i < per; ++i) loc += hs[t * per + i];
  const uint32_t excl = block_exclusive_scan<NTHR, uint32_t>(loc, warp_tot);
  if (excl < kk && kk <= excl + loc) {
    uint32_t c = excl;
#pragma unroll
    for (int i = 0; i < per; ++i) {
      const uint32_t h = hs[t * per + i];
      if (c + h >= kk) {
        res[0] = (uint32_t)(t * per + i);
        res[1] = kk - c;
        break;
      }
      c += h;
    }
  }
  __syncthreads();
}

// ---- fold kernel ---------------------------------------------------------------------
// C CTAs per group, each over a slice of the slots: fold w_prev into the scores, claim
// the fill slots (mode 1) and, for a choosing call (mode 2), add the slice's histogram of
// the top 11 key bits into the group's histogram in the workspace.
template <int NT>
__global__ void __launch_bounds__(kSelThreads, 2)
    evict_fold_kernel(const __grid_constant__ EvParams<NT> p) {
  griddep_launch_dependents();  // the choose / row kernel may be scheduled
  const int unit = blockIdx.x / p.C, rank = blockIdx.x % p.C;
  const int ti = unit / p.G, g = unit % p.G;
  const EvTarget &T = p.t[ti];
  const int tid = threadIdx.x;
  const bool choose = p.mode == 2;
  const bool vec = p.vec != 0;
  __shared__ uint32_t hs[kHistBins];
  if (choose) {
    for (int i = tid; i < kHistBins; i += kSelThreads) hs[i] = 0u;
    __syncthreads();
  }
  const int j_begin = rank * p.slice;
  const int j_end = min(p.N_C, j_begin + p.slice);
  const bool fold = T.w_prev != nullptr;
  constexpr int U = 2;
  const int stride = 4 * kSelThreads;
  for (int j0 = j_begin + 4 * tid; j0 < j_end; j0 += stride * U) {
    float ks[U][4];
    int32_t tp[U][4];
    for (int bb = 0; bb < p.nb; ++bb) {
      const size_t base = bh_of(p, g, bb) * (size_t)p.N_C;
      float sc[U][4], wp[U][4];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j4 = j0 + stride * u;
        ld4(T.scores + base, j4, j_end, vec, sc[u]);
        if (fold) ld4_cs(T.w_prev + base, j4, j_end, vec, wp[u]);
        if (bb == 0) {
          if (choose && p.need_tp)
            ld4i(T.token_pos + base, j4, j_end, vec, tp[u]);
          else {
#pragma unroll
            for (int e = 0; e < 4; ++e) tp[u][e] = 0;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j4 = j0 + stride * u;
        if (j4 >= j_end) continue;
        if (fold) {
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[u][e] = __fadd_rn(sc[u][e], wp[u][e]);
        }
        bool store = fold;
        if (p.mode == 1) {  // filling: chunk row k takes slot n_filled + k
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = j4 + e, k = j - p.n_filled;
            if (j < j_end && k >= 0 && k < p.S) {
              sc[u][e] = 0.f;
              store = true;
              const size_t gs = base + j, rk = bh_of(p, g, bb) * p.S + k;
              if (T.dpos) T.dpos[rk] = T.token_pos[gs];
              T.token_pos[gs] = p.P + k;
              if (T.slots_out) T.slots_out[rk] = j;
            }
          }
        }
        if (store) st4(T.scores + base, j4, j_end, vec, sc[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) ks[u][e] = bb == 0 ? sc[u][e] : __fadd_rn(ks[u][e], sc[u][e]);
      }
    }
    if (choose) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j4 = j0 + stride * u;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (j4 + e < j_end)
            hist_add(hs, sel_key(ks[u][e], tp[u][e], p.score_mode, p.P) >> (32 - kTopBits));
      }
    }
  }
  if (!choose) return;
  __syncthreads();
  uint32_t *gh = T.hist + (size_t)g * kHistBins;
  for (int i = tid; i < kHistBins; i += kSelThreads) {
    const uint32_t v = hs[i];
    if (v) atomicAdd(gh + i, v);
  }
}

// ---- choose kernel -------------------------------------------------------------------
// One CTA per group (mode 2), launched as a programmatic dependent of the fold kernel.
// It takes the group's histogram (and leaves zeros), finds the bin of the top 11 key bits
// holding the S-th smallest key, and then works on two bitmasks over the slots: slots
// whose key lies below that bin (all chosen) and slots whose key lies in it (the
// candidates).  The threshold is refined over the candidates only (bits 20..10, 9..0),
// the chosen candidates are added to the first mask (ties at the threshold: lowest slots
// first), and each thread lists the chosen slots of its words in slot order after one
// block scan of their counts.
//   KM 2: the group's folded h2o scores are bulk-copied into shared memory (keys formed
//         on read); KM 1: keys computed from L2 into shared memory (batch-row sums,
//         positions, unaligned capacities); KM 0: keys read from L2 each time (N_C above
//         what shared memory holds).
constexpr int kChooseThreads = 1024;
constexpr int kChooseWarps = kChooseThreads / 32;
constexpr int kMaxWordsPerThread = 2;  // 32-slot words per thread: N_C <= 65536

template <int NT>
__device__ __forceinline__ uint32_t key_from_l2(const EvParams<NT> &p, const EvTarget &T, int g,
                                                int j) {
  float ks = 0.f;
  for (int bb = 0; bb < p.nb; ++bb) {
    const float sc = __ldcg(T.scores + bh_of(p, g, bb) * p.N_C + j);
    ks = bb == 0 ? sc : __fadd_rn(ks, sc);
  }
  const int32_t tp = p.need_tp ? __ldcg(T.token_pos + bh_of(p, g, 0) * p.N_C + j) : 0;
  return sel_key(ks, tp, p.score_mode, p.P);
}

template <int NT, int KM>
__global__ void __launch_bounds__(kChooseThreads, 1)
    evict_choose_kernel(const __grid_constant__ EvParams<NT> p) {
  griddep_launch_dependents();  // the row kernel may start loading its inputs
  const int ti = blockIdx.x / p.G, g = blockIdx.x % p.G;
  const EvTarget &T = p.t[ti];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ uint32_t hs[kHistBins];
  __shared__ uint32_t hs2[kMidBins];
  __shared__ uint32_t wscan[kChooseWarps];
  __shared__ uint32_t res[4];
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t below_w[kChooseThreads * kMaxWordsPerThread];  // slots below the bin
  __shared__ uint32_t cand_w[kChooseThreads * kMaxWordsPerThread];   // slots in the bin
  extern __shared__ __align__(16) unsigned char dyn[];  // [N_C] scores or keys (KM 1, 2)
  const uint32_t keys_a = smem_u32(dyn);

  const int n_words = (p.N_C + 31) >> 5;
  if (KM == 2 && tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();  // the fold kernel's scores and histograms are complete
  uint32_t *gh = T.hist + (size_t)g * kHistBins;
  uint32_t hreg[kHistBins / kChooseThreads];
#pragma unroll
  for (int q = 0; q < kHistBins / kChooseThreads; ++q) hreg[q] = __ldcg(gh + tid + q * kChooseThreads);
  if (KM == 2 && tid == 0) {
    asm volatile("fence.proxy.async.global;" ::: "memory");
    const uint32_t bytes = (uint32_t)p.N_C * 4u;
    mbar_expect_tx(&bar, bytes);
    const unsigned char *src =
        reinterpret_cast<const unsigned char *>(T.scores + bh_of(p, g, 0) * p.N_C);
    for (uint32_t off = 0; off < bytes; off += 16384u)
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
          ::"r"(keys_a + off), "l"(src + off), "r"(bytes - off < 16384u ? bytes - off : 16384u),
          "r"(smem_u32(&bar))
          : "memory");
    mbar_arrive(&bar);
  }
#pragma unroll
  for (int q = 0; q < kHistBins / kChooseThreads; ++q) {
    hs[tid + q * kChooseThreads] = hreg[q];
    __stcg(gh + tid + q * kChooseThreads, 0u);
  }
  if (KM == 1) {
#pragma unroll 1
    for (int j = tid; j < p.N_C; j += kChooseThreads) sts32(keys_a + 4u * j, (int)key_from_l2(p, T, g, j));
  }
  __syncthreads();
  // key of slot j
#define KEY_AT(j)                                                                     \
  (KM == 2 ? order_key(__int_as_float(lds32(keys_a + 4u * (uint32_t)(j))))            \
           : KM == 1 ? (uint32_t)lds32(keys_a + 4u * (uint32_t)(j)) : key_from_l2(p, T, g, (j)))

  // ---- the bin of the top 11 bits that holds the S-th smallest key -----------------------
  find_bin<kChooseThreads, kHistBins>(hs, (uint32_t)p.S, wscan, res);
  const uint32_t top = res[0];
  uint32_t kk = res[1];
  if (KM == 2) {
    const bool ok = mbar_wait(&bar, 0, p.wait_ns);
    if (__syncthreads_or(!ok)) {  // a copy that never lands: record it, drain, give up
      if (tid == 0) {
        atomicExch(T.status, H2OKV_ERR_TIMEOUT);
        mbar_wait(&bar, 0, p.wait_ns);
      }
      __syncthreads();
      return;
    }
  }

  // ---- bitmasks: word w holds slots 32w .. 32w + 31, one per lane of a warp step; the
  // candidates' bits 20..10 are counted on the way (in a second histogram) -------------
  for (int i = tid; i < kMidBins; i += kChooseThreads) hs2[i] = 0u;
  __syncthreads();
#pragma unroll 4
  for (int w = warp; w < n_words; w += kChooseWarps) {
    const int j = 32 * w + lane;
    const bool okj = j < p.N_C;
    const uint32_t key = okj ? KEY_AT(j) : 0xffffffffu;
    const uint32_t b = okj ? key >> (32 - kTopBits) : 0xffffffffu;
    const uint32_t bm = __ballot_sync(0xffffffffu, b < top);
    const uint32_t cm = __ballot_sync(0xffffffffu, b == top);
    if (lane == 0) {
      below_w[w] = bm;
      cand_w[w] = cm;
    }
    if (b == top) hist_add(hs2, (key >> 10) & 2047u);
  }
  __syncthreads();

  // ---- threshold: bits 20..10, then 9..0, of the candidates ------------------------------
  // thread t owns words t * wpt .. t * wpt + wpt - 1 (slot order follows thread order)
  const int wpt = (n_words + kChooseThreads - 1) / kChooseThreads;
  find_bin<kChooseThreads, kMidBins>(hs2, kk, wscan, res);
  const uint32_t pre = (top << 11) | res[0];  // key bits 31..10
  kk = res[1];
  for (int i = tid; i < kLowBins; i += kChooseThreads) hs[i] = 0u;
  __syncthreads();
#pragma unroll
  for (int q = 0; q < kMaxWordsPerThread; ++q) {
    const int w = tid * wpt + q;
    if (q >= wpt || w >= n_words) break;
    for (uint32_t m = cand_w[w]; m; m &= m - 1u) {
      const uint32_t key = KEY_AT(32 * w + __ffs(m) - 1);
      if ((key >> 10) == pre) hist_add(hs, key & 1023u);
    }
  }
  __syncthreads();
  find_bin<kChooseThreads, kLowBins>(hs, kk, wscan, res);
  const uint32_t Tk = (pre << 10) | res[0];  // take every key < Tk and the first k_eq keys == Tk
  const uint32_t k_eq = res[1];

  // ---- chosen words: below the bin, candidates < Tk, the first k_eq candidates == Tk -----
  uint32_t lt[kMaxWordsPerThread], eq[kMaxWordsPerThread];
  uint32_t n_eq = 0;
#pragma unroll
  for (int q = 0; q < kMaxWordsPerThread; ++q) {
    lt[q] = 0u;
    eq[q] = 0u;
    const int w = tid * wpt + q;
    if (q >= wpt || w >= n_words) continue;
    lt[q] = below_w[w];
    for (uint32_t m = cand_w[w]; m; m &= m - 1u) {
      const int bit = __ffs(m) - 1;
      const uint32_t key = KEY_AT(32 * w + bit);
      if (key < Tk) lt[q] |= 1u << bit;
      else if (key == Tk) eq[q] |= 1u << bit;
    }
    n_eq += __popc(eq[q]);
  }
  uint32_t eb = block_exclusive_scan<kChooseThreads, uint32_t>(n_eq, wscan);
  uint32_t n_take = 0;
#pragma unroll
  for (int q = 0; q < kMaxWordsPerThread; ++q) {
    for (uint32_t m = eq[q]; m && eb < k_eq; m &= m - 1u, ++eb) lt[q] |= m & (0u - m);
    n_take += __popc(lt[q]);
  }
  uint32_t pos = block_exclusive_scan<kChooseThreads, uint32_t>(n_take, wscan);

  // ---- the chosen slots in slot order (the row kernel claims them) -----------------------
  int32_t *slist = T.slotlist + (size_t)g * p.S;
#pragma unroll
  for (int q = 0; q < kMaxWordsPerThread; ++q) {
    const int w = tid * wpt + q;
    for (uint32_t m = lt[q]; m; m &= m - 1u, ++pos) __stcg(slist + pos, 32 * w + __ffs(m) - 1);
  }
}
#undef KEY_AT

// ---- row kernel ----------------------------------------------------------------------
// blockIdx.y = row set = (cache, group, batch row in the group); blockIdx.x covers the
// set's S chunk rows, key and value.
template <int NT>
struct RowSet {
  const EvTarget *T;
  size_t bh;        // (batch row, KV head) index of the set
  int32_t *slist;   // the group's chosen slots (mode 2)
};
template <int NT>
__device__ __forceinline__ RowSet<NT> row_set(const EvParams<NT> &p) {
  const int set = blockIdx.y;
  const int bb = set % p.nb, ug = set / p.nb;
  const int g = ug % p.G, ti = ug / p.G;
  RowSet<NT> r;
  r.T = &p.t[ti];
  r.bh = bh_of(p, g, bb);
  r.slist = p.t[ti].slotlist + (size_t)g * p.S;
  return r;
}

// Slot of chunk row k of a set (negative: skipped -- a replayed slot outside the cache).
template <int NT>
__device__ __forceinline__ int slot_of(const EvParams<NT> &p, const RowSet<NT> &rs, int k) {
  if (p.mode == 1) return p.n_filled + k;
  if (p.mode == 2) return __ldcg(rs.slist + k);  // in range: zeroed on create, written by choose
  const int j = __ldg(rs.T->slots_in + rs.bh * p.S + k);
  return (j >= 0 && j < p.N_C) ? j : -1;
}

// The bookkeeping of a chosen (mode 2) or logged (mode 3) slot, once per chunk row with
// its key row: old position to the delta output, new position, score 0, slot list out.
template <int NT>
__device__ __forceinline__ void row_claim(const EvParams<NT> &p, const RowSet<NT> &rs, int k,
                                          int j) {
  const EvTarget &T = *rs.T;
  if (j < 0) {
    atomicExch(T.status, H2OKV_ERR_INVALID_ARG);
    return;
  }
  const size_t gs = rs.bh * p.N_C + j, rk = rs.bh * p.S + k;
  if (T.dpos) __stcg(T.dpos + rk, __ldcg(T.token_pos + gs));
  __stcg(T.token_pos + gs, p.P + k);
  __stcg(T.scores + gs, 0.f);
  if (p.mode == 2 && T.slots_out) __stcg(T.slots_out + rk, j);
}

// f32 / bf16 caches: the set's rows are cut into 16-byte pieces (e = (2k + t) * PC + c),
// consecutive threads take consecutive pieces, every thread keeps kCopyUnroll pieces in
// flight.  The first pieces are loaded before the wait on the select kernel.
template <int NT, bool DELTA>
__device__ __forceinline__ void copy_rows(const EvParams<NT> &p) {
  const RowSet<NT> rs = row_set(p);
  const EvTarget &T = *rs.T;
  const int PC = p.row_bytes / 16;
  const int total = p.S * 2 * PC;
  const int nthr = gridDim.x * kRowThreads;
  const int first = blockIdx.x * kRowThreads + threadIdx.x;
  const uint4 *src_k = reinterpret_cast<const uint4 *>(T.k_new + rs.bh * p.S * (size_t)p.in_row_bytes);
  const uint4 *src_v = reinterpret_cast<const uint4 *>(T.v_new + rs.bh * p.S * (size_t)p.in_row_bytes);
  uint4 *dst_k = reinterpret_cast<uint4 *>(T.keys + rs.bh * p.N_C * (size_t)p.row_bytes);
  uint4 *dst_v = reinterpret_cast<uint4 *>(T.values + rs.bh * p.N_C * (size_t)p.row_bytes);
  uint4 r[kCopyUnroll];
  int rr[kCopyUnroll];  // 2k + t of each piece (-1: none)
  int cc[kCopyUnroll];
  auto load = [&](int base) {
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const int e = base + u * nthr;
      rr[u] = -1;
      if (e < total) {
        rr[u] = e / PC;
        cc[u] = e - rr[u] * PC;
        r[u] = __ldcs(((rr[u] & 1) ? src_v : src_k) + (size_t)(rr[u] >> 1) * PC + cc[u]);
      }
    }
  };
  load(first);
  griddep_wait();
  for (int base = first; base < total; base += nthr * kCopyUnroll) {
    if (base != first) load(base);
    int slot[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) slot[u] = rr[u] >= 0 ? slot_of(p, rs, rr[u] >> 1) : -1;
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      if (rr[u] < 0) continue;
      const int k = rr[u] >> 1, t = rr[u] & 1;
      if (p.mode >= 2 && t == 0 && cc[u] == 0) row_claim(p, rs, k, slot[u]);
      if (slot[u] < 0) continue;
      uint4 *dst = (t ? dst_v : dst_k) + (size_t)slot[u] * PC + cc[u];
      if (DELTA && T.dk) {
        uint4 *dd = reinterpret_cast<uint4 *>((t ? T.dv : T.dk) + (rs.bh * p.S + k) * (size_t)p.row_bytes);
        __stcg(dd + cc[u], __ldcg(dst));
      }
      __stcg(dst, r[u]);
    }
  }
}

// int8 / int4 caches: one row per segment of L lanes (L = the smallest power of two >=
// d / 32); lane i of a segment holds the 8-element chunks i, i + L, ... (up to four) of
// the row, so the per-row work (absmax reduction, IEEE division by qmax, fp16 scale,
// correctly rounded reciprocal, addressing, the slot's bookkeeping) is shared by up to
// 32 elements per lane.  Per row, the same arithmetic as the per-row quantizer:
// absmax, IEEE division by qmax, clamp to the fp16 range, round to fp16, then the code
// of quant_code (in pairs).
__host__ __device__ __forceinline__ int quant_lanes(int d) {
  const int g8 = d / 8;
  const int need = (g8 + kQuantChunks - 1) / kQuantChunks;
  int L = 1;
  while (L < need) L <<= 1;
  return L;
}

template <int NT, int KV, bool DELTA>
__device__ __forceinline__ void quantize_rows(const EvParams<NT> &p) {
  constexpr int qmax = KV == H2OKV_I8 ? 127 : 7;
  const RowSet<NT> rs = row_set(p);
  const EvTarget &T = *rs.T;
  const int G8 = p.d / 8;
  const int L = quant_lanes(p.d);
  const int lane = threadIdx.x & 31;
  const int seg = lane / L, li = lane % L, segs = 32 / L;
  const int items = p.S * 2;  // (chunk row k, t) as 2k + t: t = 0 key row, 1 value row
  const int W = gridDim.x * kRowWarps;
  const int w0 = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  const uint8_t *src_k = T.k_new + rs.bh * p.S * (size_t)p.in_row_bytes;
  const uint8_t *src_v = T.v_new + rs.bh * p.S * (size_t)p.in_row_bytes;
  uint4 xr[kQuantUnroll][kQuantChunks];
  auto item_of = [&](int base, int u) { return ((base + u * W) * segs) + seg; };
  auto load = [&](int base) {
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int it = item_of(base, u);
      const uint4 *src = reinterpret_cast<const uint4 *>(((it & 1) ? src_v : src_k) +
                                                         (size_t)(it >> 1) * p.in_row_bytes);
#pragma unroll
      for (int c = 0; c < kQuantChunks; ++c) {
        const int ch = li + c * L;
        xr[u][c] = make_uint4(0u, 0u, 0u, 0u);
        if (it < items && ch < G8) xr[u][c] = __ldcs(src + ch);
      }
    }
  };
  load(w0);
  griddep_wait();
  for (int base = w0; base * segs < items; base += W * kQuantUnroll) {
    if (base != w0) load(base);
    int slot[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int it = item_of(base, u);
      slot[u] = it < items ? slot_of(p, rs, it >> 1) : -1;
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int it = item_of(base, u);
      float amax = 0.f;  // the zero-filled chunks past the row do not change it
#pragma unroll
      for (int c = 0; c < kQuantChunks; ++c) {
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&xr[u][c]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(h2[q]);
          amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
      for (int o = L >> 1; o > 0; o >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      float rq = amax / (float)qmax;  // IEEE division
      rq = fminf(rq, 65504.f);
      const __half hs = __float2half_rn(rq);
      const float s = __half2float(hs);
      const float y = __frcp_rn(s);
      const bool nz = s > 0.f;  // scale 0: every code 0
      if (it >= items) continue;
      const int t = it & 1, k = it >> 1;
      const int j = slot[u];
      if (p.mode >= 2 && t == 0 && li == 0) row_claim(p, rs, k, j);
      if (j < 0) continue;
      const size_t drow = rs.bh * p.N_C + j, crow = rs.bh * p.S + k;
      uint8_t *codes = (t ? T.values : T.keys) + drow * (size_t)p.row_bytes;
      __half *sdst = (t ? T.v_scales : T.k_scales) + drow;
      if (DELTA && T.dk) {
        uint8_t *dcodes = (t ? T.dv : T.dk) + crow * (size_t)p.row_bytes;
        if (li == 0) (t ? T.dvs : T.dks)[crow] = *sdst;
#pragma unroll
        for (int c = 0; c < kQuantChunks; ++c) {
          const int ch = li + c * L;
          if (ch >= G8) break;
          if (KV == H2OKV_I8)
            reinterpret_cast<uint2 *>(dcodes)[ch] = __ldcg(reinterpret_cast<const uint2 *>(codes) + ch);
          else
            reinterpret_cast<uint32_t *>(dcodes)[ch] =
                __ldcg(reinterpret_cast<const unsigned int *>(codes) + ch);
        }
      }
      if (li == 0) *sdst = hs;
#pragma unroll
      for (int c = 0; c < kQuantChunks; ++c) {
        const int ch = li + c * L;
        if (ch >= G8) break;
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&xr[u][c]);
        uint2 bits[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) bits[q] = quant_bits2(__bfloat1622float2(h2[q]), s, y, (float)qmax);
        if (KV == H2OKV_I8) {
          uint32_t lo = 0u, hi = 0u;  // code bytes: the low byte of each rounded value
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            lo |= ((bits[q].x & 0xFFu) | ((bits[q].y & 0xFFu) << 8)) << (16 * q);
            hi |= ((bits[q + 2].x & 0xFFu) | ((bits[q + 2].y & 0xFFu) << 8)) << (16 * q);
          }
          __stcg(reinterpret_cast<uint2 *>(codes) + ch, nz ? make_uint2(lo, hi) : make_uint2(0u, 0u));
        } else {
          uint32_t w = 0u;  // element 2i in the low nibble of byte i
#pragma unroll
          for (int q = 0; q < 4; ++q)
            w |= ((bits[q].x & 0xFu) | ((bits[q].y & 0xFu) << 4)) << (8 * q);
          __stcg(reinterpret_cast<unsigned int *>(codes) + ch, nz ? w : 0u);
        }
      }
    }
  }
}

template <int NT, int KV, bool DELTA>
__global__ void __launch_bounds__(kRowThreads) evict_rows_kernel(const __grid_constant__ EvParams<NT> p) {
  if constexpr (KV == H2OKV_I8 || KV == H2OKV_I4)
    quantize_rows<NT, KV, DELTA>(p);
  else
    copy_rows<NT, DELTA>(p);
}

// ---- per-row quantizer (kv_cache_quantize) ---------------------------------------------
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
  const float y = __frcp_rn(s);
  for (int p = lane; p < d / 2; p += 32) {
    const float2 v = __bfloat1622float2(x2[p]);
    int qa = 0, qb = 0;
    if (s > 0.f) {
      qa = quant_code(v.x, s, y, (float)qmax);
      qb = quant_code(v.y, s, y, (float)qmax);
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

// ---- launch --------------------------------------------------------------------------
// Everything of a call that the caches share (they must agree on it).
struct EvCall {
  int mode, S, P, n_filled, score_mode;
  bool orig, delta;
};

EvTarget target_of(h2okv_cache *c, const float *w_prev, const void *k_new, const void *v_new,
                   int32_t *slots_out, const int32_t *slots_in, const h2okv_delta *delta) {
  uint8_t *ws = reinterpret_cast<uint8_t *>(c->bufs.workspace);
  EvTarget t;
  t.scores = c->bufs.scores;
  t.w_prev = w_prev;
  t.token_pos = c->bufs.token_pos;
  t.k_new = reinterpret_cast<const uint8_t *>(k_new);
  t.v_new = reinterpret_cast<const uint8_t *>(v_new);
  t.keys = reinterpret_cast<uint8_t *>(c->bufs.keys);
  t.values = reinterpret_cast<uint8_t *>(c->bufs.values);
  t.k_scales = reinterpret_cast<__half *>(c->bufs.k_scales);
  t.v_scales = reinterpret_cast<__half *>(c->bufs.v_scales);
  t.slots_out = slots_out;
  t.slots_in = slots_in;
  t.dk = delta ? reinterpret_cast<uint8_t *>(delta->keys) : nullptr;
  t.dv = delta ? reinterpret_cast<uint8_t *>(delta->values) : nullptr;
  t.dks = delta ? reinterpret_cast<__half *>(delta->k_scales) : nullptr;
  t.dvs = delta ? reinterpret_cast<__half *>(delta->v_scales) : nullptr;
  t.dpos = delta ? delta->token_pos : nullptr;
  t.hist = reinterpret_cast<uint32_t *>(ws + c->ws.ev_hist);
  t.arrive = reinterpret_cast<uint32_t *>(ws + c->ws.ev_arrive);
  t.slotlist = reinterpret_cast<int32_t *>(ws + c->ws.ev_slots);
  t.status = reinterpret_cast<int *>(ws + c->ws.status);
  return t;
}

// Shared-memory opt-in of one choose kernel instance, once per device.
template <int NT, int KM>
int opt_in_choose() {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(H2OKV_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(
        evict_choose_kernel<NT, KM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
        (int)(kSmemKeysMax * 4));
    if (e != cudaSuccess)
      return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(evict_choose_kernel): %s",
                       cudaGetErrorString(e));
    done[dev] = true;
  }
  return H2OKV_OK;
}

template <int NT, int KV>
int launch_rows(const EvParams<NT> &p, bool delta, int sms, cudaStream_t st) {
  const long long sets = (long long)p.n_targets * p.G * p.nb;
  long long work;  // independent units of one set (pieces, or lane segments)
  int per_cta;
  if (KV == H2OKV_I8 || KV == H2OKV_I4) {
    work = (long long)p.S * 2;
    per_cta = kRowWarps * (32 / quant_lanes(p.d)) * kQuantUnroll;
  } else {
    work = (long long)p.S * 2 * (p.row_bytes / 16);
    per_cta = kRowThreads * kCopyUnroll;
  }
  if (work <= 0 || sets <= 0) return H2OKV_OK;
  if (sets > 65535 || work >= (1LL << 30))
    return set_error(H2OKV_ERR_UNSUPPORTED, "too many chunk rows in one eviction call");
  // CTAs per set: every row of the call in flight in one round (CTAs are cheap; a CTA
  // that looped over many rounds would wait on memory once per round)
  const long long gx = (work + per_cta - 1) / per_cta;
  if (gx > 65535) return set_error(H2OKV_ERR_UNSUPPORTED, "chunk too long for one eviction call");
  (void)sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)gx, (unsigned)sets);
  cfg.blockDim = dim3(kRowThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = delta ? cudaLaunchKernelEx(&cfg, evict_rows_kernel<NT, KV, true>, p)
                        : cudaLaunchKernelEx(&cfg, evict_rows_kernel<NT, KV, false>, p);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "evict_rows_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("evict_rows_kernel");
}

template <int NT>
int launch_evict_t(h2okv_cache *const *caches, int n, const EvTarget *targets, const EvCall &call,
                   cudaStream_t st) {
  const h2okv_cache_desc &d = caches[0]->desc;
  EvParams<NT> p;
  for (int i = 0; i < n; ++i) p.t[i] = targets[i];
  p.n_targets = n;
  p.nb = call.orig ? d.batch : 1;
  p.G = call.orig ? d.n_kv_heads : d.batch * d.n_kv_heads;
  p.Hk = d.n_kv_heads;
  p.N_C = d.capacity;
  p.S = call.S;
  p.P = call.P;
  p.n_filled = call.n_filled;
  p.d = d.head_dim;
  p.mode = call.mode;
  p.score_mode = call.score_mode;
  p.need_tp = (call.n_filled < d.capacity || call.score_mode == H2OKV_SCORE_H2O_NORM) ? 1 : 0;
  p.vec = d.capacity % 4 == 0 ? 1 : 0;
  p.row_bytes = (int)caches[0]->row_bytes;
  p.in_row_bytes = d.head_dim * (d.q_dtype == H2OKV_F32 ? 4 : 2);
  p.wait_ns = caches[0]->wait_timeout_ns;
  const int sms = caches[0]->sms > 0 ? caches[0]->sms : 148;
  const int units = n * p.G;
  // fold CTAs per group: about four per SM in all, slices of at least 2048 slots
  const int by_sm = max(1, (4 * sms) / units);
  const int by_len = max(1, (d.capacity + 2047) / 2048);
  p.C = min(by_sm, by_len);
  p.slice = ((d.capacity + p.C - 1) / p.C + 3) & ~3;
  p.C = (d.capacity + p.slice - 1) / p.slice;
  if ((long long)units * p.C > INT32_MAX)
    return set_error(H2OKV_ERR_UNSUPPORTED, "too many groups in one eviction call");
  evict_fold_kernel<NT><<<units * p.C, kSelThreads, 0, st>>>(p);
  int rc = check_launch("evict_fold_kernel");
  if (rc || p.mode == 0) return rc;
  if (p.mode == 2) {
    // key source of the choose kernel (see there)
    const bool fits = d.capacity <= kSmemKeysMax;
    const int km = !fits ? 0
                   : (p.vec && p.nb == 1 && !p.need_tp && p.score_mode != H2OKV_SCORE_H2O_NORM) ? 2
                                                                                            : 1;
    const size_t smem = fits ? (size_t)d.capacity * 4 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)units);
    cfg.blockDim = dim3(kChooseThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (km == 2) {
      rc = opt_in_choose<NT, 2>();
      if (rc) return rc;
      e = cudaLaunchKernelEx(&cfg, evict_choose_kernel<NT, 2>, p);
    } else if (km == 1) {
      rc = opt_in_choose<NT, 1>();
      if (rc) return rc;
      e = cudaLaunchKernelEx(&cfg, evict_choose_kernel<NT, 1>, p);
    } else {
      rc = opt_in_choose<NT, 0>();
      if (rc) return rc;
      e = cudaLaunchKernelEx(&cfg, evict_choose_kernel<NT, 0>, p);
    }
    if (e != cudaSuccess)
      return set_error(H2OKV_ERR_CUDA, "evict_choose_kernel launch: %s", cudaGetErrorString(e));
    rc = check_launch("evict_choose_kernel");
    if (rc) return rc;
  }
  switch (d.kv_dtype) {
    case H2OKV_F32: return launch_rows<NT, H2OKV_F32>(p, call.delta, sms, st);
    case H2OKV_BF16: return launch_rows<NT, H2OKV_BF16>(p, call.delta, sms, st);
    case H2OKV_I8: return launch_rows<NT, H2OKV_I8>(p, call.delta, sms, st);
    case H2OKV_I4: return launch_rows<NT, H2OKV_I4>(p, call.delta, sms, st);
  }
  return set_error(H2OKV_ERR_UNSUPPORTED, "kv dtype");
}

constexpr int kMaxCachesPerLaunch = 48;

}  // namespace

int launch_init_cache(h2okv_cache *c, cudaStream_t st) {
  const size_t n = (size_t)c->desc.batch * c->desc.n_kv_heads * c->desc.capacity;
  uint8_t *ws = reinterpret_cast<uint8_t *>(c->bufs.workspace);
  if (cudaMemsetAsync(ws + c->ws.status, 0, 4, st) != cudaSuccess ||
      cudaMemsetAsync(ws + c->ws.ev_hist, 0, c->ws.ev_zero_end - c->ws.ev_hist, st) != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaMemsetAsync(workspace) failed");
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  init_kernel<<<blocks, 256, 0, st>>>(c->bufs.token_pos, c->bufs.scores, n);
  return check_launch("init_kernel");
}

// Mode of a call on a cache in this state.
static int call_mode(const h2okv_cache *c, int S, const int32_t *slots_in) {
  return S == 0 ? 0 : (slots_in ? 3 : (c->n_filled + S <= c->desc.capacity ? 1 : 2));
}

int launch_evict_insert(h2okv_cache *c, const float *w_prev, const void *k_new, const void *v_new,
                        int S, int64_t P, int32_t *slots_out, const int32_t *slots_in,
                        const h2okv_delta *delta, cudaStream_t st) {
  EvCall call;
  call.mode = call_mode(c, S, slots_in);
  call.S = S;
  call.P = (int)P;
  call.n_filled = c->n_filled;
  call.score_mode = c->score_mode;
  // h2o_orig: one group per KV head chooses for every batch row
  call.orig = c->score_mode == H2OKV_SCORE_H2O_ORIG && call.mode == 2;
  call.delta = delta != nullptr;
  const EvTarget t = target_of(c, w_prev, k_new, v_new, slots_out, slots_in, delta);
  return launch_evict_t<1>(&c, 1, &t, call, st);
}

int launch_evict_insert_many(h2okv_cache *const *caches, int n, const float *const *w_prev,
                             const void *const *k_new, const void *const *v_new, int S, int64_t P,
                             int32_t *const *slots_out, cudaStream_t st) {
  const h2okv_cache *c0 = caches[0];
  EvCall call;
  call.mode = call_mode(c0, S, nullptr);
  call.S = S;
  call.P = (int)P;
  call.n_filled = c0->n_filled;
  call.score_mode = c0->score_mode;
  call.orig = c0->score_mode == H2OKV_SCORE_H2O_ORIG && call.mode == 2;
  call.delta = false;
  EvTarget t[kMaxCachesPerLaunch];
  for (int base = 0; base < n; base += kMaxCachesPerLaunch) {
    const int m = min(kMaxCachesPerLaunch, n - base);
    for (int i = 0; i < m; ++i)
      t[i] = target_of(caches[base + i], w_prev ? w_prev[base + i] : nullptr,
                       k_new ? k_new[base + i] : nullptr, v_new ? v_new[base + i] : nullptr,
                       slots_out ? slots_out[base + i] : nullptr, nullptr, nullptr);
    const int rc = m == 1 ? launch_evict_t<1>(caches + base, 1, t, call, st)
                          : launch_evict_t<kMaxCachesPerLaunch>(caches + base, m, t, call, st);
    if (rc) return rc;
  }
  return H2OKV_OK;
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
