// Gradients of a chunk's SDPA over the cache ("Learning how to Forget", §A.5: the
// backward pass runs autograd over each chunk's computation while the cache
// policy's decisions are replayed, not differentiated).  For query head h of
// group g, row i (token P + i) and slot j:
//   s_ij = q_i . k_j / sqrt(d), p_ij = exp(s_ij - lse_i) (0 where P + i < t_j),
//   dP_ij = dy_i . v_j,  D_i = sum_j p_ij dP_ij,  dS_ij = p_ij (dP_ij - D_i),
//   dq_i = sum_j dS_ij k_j / sqrt(d),
//   dk_j = sum over the group's heads and rows of dS_ij q_i / sqrt(d),
//   dv_j = sum over the group's heads and rows of p_ij dy_i.
// lse is the forward's natural-log row log-sum-exp.  A bf16 cache with d = 128 and bf16
// queries goes to the tensor-core kernels of attn_bwd_tc.cu; every other combination
// runs here, on CUDA cores, in float32:
//   bwd_rows_kernel   one CTA per 32 packed rows of a group: pass 1 finds D_i,
//                     pass 2 accumulates dq_i (no atomics);
//   bwd_slots_kernel  one CTA per 32 slots of a group: streams every packed row of
//                     the group and accumulates dk_j, dv_j (no atomics).
// Both use the same tiling: 32 x 32 (row, slot) blocks, dot products by lanes over
// padded shared-memory rows, accumulations by lanes over head-dimension columns.
#include <math.h>

#include "h2okv_internal.cuh"

namespace h2okv {
namespace {

constexpr int kT = 32;         // rows / slots per tile
constexpr int kBwdThreads = 256;
constexpr int kCols = kMaxHeadDim / 32;

template <int KV>
__device__ __forceinline__ float load_cache(const uint8_t *__restrict__ row, const __half *scale,
                                            int e) {
  if constexpr (KV == H2OKV_F32) {
    return reinterpret_cast<const float *>(row)[e];
  } else if constexpr (KV == H2OKV_BF16) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(row)[e]);
  } else if constexpr (KV == H2OKV_I8) {
    return (float)(int8_t)row[e] * __half2float(*scale);
  } else {
    const uint8_t b = row[e >> 1];
    int v = (e & 1) ? (b >> 4) : (b & 0xF);
    v = v >= 8 ? v - 16 : v;
    return (float)v * __half2float(*scale);
  }
}

template <int QT>
__device__ __forceinline__ float load_in(const void *p, size_t idx) {
  if constexpr (QT == H2OKV_F32)
    return reinterpret_cast<const float *>(p)[idx];
  else
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[idx]);
}

struct BwdArgs {
  const void *q, *dy;
  const float *lse;
  const uint8_t *keys, *values;
  const __half *k_scales, *v_scales;
  const int32_t *token_pos;
  float *dq, *dk, *dv, *D;
  int Hq, Hk, q_g, d, N_C, S, P;
  size_t row_bytes;
  float c2;     // log2(e) / sqrt(d)
  float rsd;    // 1 / sqrt(d)
};

// shared memory (floats): two row tiles [kT][d+1] (q, dy), two slot tiles [kT][d+1]
// (k, v), two (row, slot) tiles [kT][kT+1] (p, dS), slot positions, row lse / D
__host__ __device__ inline size_t bwd_smem_bytes(int d) {
  return 4 * (4 * (size_t)kT * (d + 1) + 2 * (size_t)kT * (kT + 1) + 3 * kT);
}

// Packed row r of group (b, g): head g * q_g + r / S, chunk row r % S.
struct RowRef {
  bool ok;
  int i;
  size_t lin;  // (b * Hq + h) * S + i
};
__device__ __forceinline__ RowRef row_ref(const BwdArgs &a, int b, int g, int r) {
  RowRef x;
  x.ok = r < a.q_g * a.S;
  const int rr = x.ok ? r : 0;
  const int h = g * a.q_g + rr / a.S;
  x.i = rr % a.S;
  x.lin = (size_t)(b * a.Hq + h) * a.S + x.i;
  return x;
}

template <int QT>
__device__ __forceinline__ void stage_rows(const BwdArgs &a, int b, int g, int r0, float *qs,
                                           float *dys, float *ls, float *Ds, bool want_D) {
  const int d = a.d;
  for (int idx = threadIdx.x; idx < kT * d; idx += kBwdThreads) {
    const int rr = idx / d, e = idx - rr * d;
    const RowRef x = row_ref(a, b, g, r0 + rr);
    qs[rr * (d + 1) + e] = x.ok ? load_in<QT>(a.q, x.lin * d + e) : 0.f;
    dys[rr * (d + 1) + e] = x.ok ? load_in<QT>(a.dy, x.lin * d + e) : 0.f;
  }
  if (threadIdx.x < kT) {
    const RowRef x = row_ref(a, b, g, r0 + threadIdx.x);
    ls[threadIdx.x] = x.ok ? a.lse[x.lin] : -INFINITY;
    if (want_D) Ds[threadIdx.x] = x.ok ? a.D[x.lin] : 0.f;
  }
}

template <int KV>
__device__ __forceinline__ void stage_slots(const BwdArgs &a, size_t slot0, int t0, float *ks,
                                            float *vs, int *tps) {
  const int d = a.d;
  const uint8_t *kb = a.keys + slot0 * a.row_bytes, *vb = a.values + slot0 * a.row_bytes;
  const __half *ksc = a.k_scales ? a.k_scales + slot0 : nullptr;
  const __half *vsc = a.v_scales ? a.v_scales + slot0 : nullptr;
  for (int idx = threadIdx.x; idx < kT * d; idx += kBwdThreads) {
    const int jj = idx / d, e = idx - jj * d;
    const int j = t0 + jj;
    float kv = 0.f, vv = 0.f;
    if (j < a.N_C) {
      kv = load_cache<KV>(kb + (size_t)j * a.row_bytes, ksc ? ksc + j : nullptr, e);
      vv = load_cache<KV>(vb + (size_t)j * a.row_bytes, vsc ? vsc + j : nullptr, e);
    }
    ks[jj * (d + 1) + e] = kv;
    vs[jj * (d + 1) + e] = vv;
  }
  if (threadIdx.x < kT)
    tps[threadIdx.x] = (t0 + threadIdx.x < a.N_C) ? a.token_pos[slot0 + t0 + threadIdx.x] : kEmptyPos;
}

// ---- dq and D: rows stationary -------------------------------------------------------
template <int QT, int KV>
__global__ void __launch_bounds__(kBwdThreads) bwd_rows_kernel(BwdArgs a) {
  extern __shared__ float sm[];
  const int d = a.d;
  float *qs = sm, *dys = qs + kT * (d + 1), *ks = dys + kT * (d + 1), *vs = ks + kT * (d + 1);
  float *ps = vs + kT * (d + 1), *dss = ps + kT * (kT + 1);
  int *tps = reinterpret_cast<int *>(dss + kT * (kT + 1));
  float *ls = reinterpret_cast<float *>(tps + kT), *Ds = ls + kT;
  const int bg = blockIdx.y, b = bg / a.Hk, g = bg - b * a.Hk;
  const int r0 = blockIdx.x * kT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t slot0 = (size_t)bg * a.N_C;

  stage_rows<QT>(a, b, g, r0, qs, dys, ls, Ds, false);
  RowRef rw[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) rw[q] = row_ref(a, b, g, r0 + warp * 4 + q);
  float Dp[4] = {0.f, 0.f, 0.f, 0.f};
  float acc[4][kCols];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < kCols; ++c) acc[q][c] = 0.f;

  for (int pass = 0; pass < 2; ++pass) {
    if (pass == 1) {
      // D_i of the warp's rows, summed over the lanes (slots)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v = Dp[q];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) Ds[warp * 4 + q] = v;
        if (lane == 0 && rw[q].ok) a.D[rw[q].lin] = v;
      }
    }
    for (int t0 = 0; t0 < a.N_C; t0 += kT) {
      __syncthreads();  // previous tile consumed (and D visible)
      stage_slots<KV>(a, slot0, t0, ks, vs, tps);
      __syncthreads();
      // lane = slot of the tile, 4 rows per warp: logits and dy . v
      float s[4] = {0.f, 0.f, 0.f, 0.f}, dp[4] = {0.f, 0.f, 0.f, 0.f};
      const float *krow = ks + lane * (d + 1), *vrow = vs + lane * (d + 1);
      for (int e = 0; e < d; ++e) {
        const float kv = krow[e], vv = vrow[e];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          s[q] = fmaf(qs[(warp * 4 + q) * (d + 1) + e], kv, s[q]);
          dp[q] = fmaf(dys[(warp * 4 + q) * (d + 1) + e], vv, dp[q]);
        }
      }
      const int tpj = tps[lane];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float l = ls[warp * 4 + q];
        const bool vis = rw[q].ok && l != -INFINITY && (int64_t)tpj <= (int64_t)a.P + rw[q].i;
        const float p = vis ? exp2f(s[q] * a.c2 - l * 1.4426950408889634f) : 0.f;
        if (pass == 0) {
          Dp[q] = fmaf(p, dp[q], Dp[q]);
        } else {
          dss[(warp * 4 + q) * (kT + 1) + lane] = p * (dp[q] - Ds[warp * 4 + q]);
        }
      }
      if (pass == 1) {
        __syncwarp();
        // dq of the warp's rows: lane = head-dimension column, sum over the tile's slots
        for (int jj = 0; jj < kT; ++jj) {
#pragma unroll
          for (int c = 0; c < kCols; ++c) {
            const int e = lane + 32 * c;
            if (e < d) {
              const float kv = ks[jj * (d + 1) + e];
#pragma unroll
              for (int q = 0; q < 4; ++q)
                acc[q][c] = fmaf(dss[(warp * 4 + q) * (kT + 1) + jj], kv, acc[q][c]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (!rw[q].ok) continue;
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const int e = lane + 32 * c;
      if (e < d) a.dq[rw[q].lin * d + e] = acc[q][c] * a.rsd;
    }
  }
}

// ---- dk and dv: slots stationary ------------------------------------------------------
template <int QT, int KV>
__global__ void __launch_bounds__(kBwdThreads) bwd_slots_kernel(BwdArgs a) {
  extern __shared__ float sm[];
  const int d = a.d;
  float *qs = sm, *dys = qs + kT * (d + 1), *ks = dys + kT * (d + 1), *vs = ks + kT * (d + 1);
  float *ps = vs + kT * (d + 1), *dss = ps + kT * (kT + 1);
  int *tps = reinterpret_cast<int *>(dss + kT * (kT + 1));
  float *ls = reinterpret_cast<float *>(tps + kT), *Ds = ls + kT;
  const int bg = blockIdx.y, b = bg / a.Hk, g = bg - b * a.Hk;
  const int t0 = blockIdx.x * kT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t slot0 = (size_t)bg * a.N_C;
  const int n_packed = a.q_g * a.S;

  stage_slots<KV>(a, slot0, t0, ks, vs, tps);
  float adk[4][kCols], adv[4][kCols];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < kCols; ++c) adk[q][c] = adv[q][c] = 0.f;

  for (int r0 = 0; r0 < n_packed; r0 += kT) {
    __syncthreads();  // previous row tile consumed
    stage_rows<QT>(a, b, g, r0, qs, dys, ls, Ds, true);
    __syncthreads();
    // lane = packed row of the tile, 4 slots per warp: logits and dy . v
    const RowRef x = row_ref(a, b, g, r0 + lane);
    float s[4] = {0.f, 0.f, 0.f, 0.f}, dp[4] = {0.f, 0.f, 0.f, 0.f};
    const float *qrow = qs + lane * (d + 1), *dyrow = dys + lane * (d + 1);
    for (int e = 0; e < d; ++e) {
      const float qv = qrow[e], dyv = dyrow[e];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        s[q] = fmaf(ks[(warp * 4 + q) * (d + 1) + e], qv, s[q]);
        dp[q] = fmaf(vs[(warp * 4 + q) * (d + 1) + e], dyv, dp[q]);
      }
    }
    const float l = ls[lane], Dl = Ds[lane];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int jj = warp * 4 + q;
      const bool vis = x.ok && l != -INFINITY && t0 + jj < a.N_C &&
                       (int64_t)tps[jj] <= (int64_t)a.P + x.i;
      const float p = vis ? exp2f(s[q] * a.c2 - l * 1.4426950408889634f) : 0.f;
      ps[jj * (kT + 1) + lane] = p;
      dss[jj * (kT + 1) + lane] = p * (dp[q] - Dl);
    }
    __syncwarp();
    // dk, dv of the warp's slots: lane = head-dimension column, sum over the tile's rows
    for (int rr = 0; rr < kT; ++rr) {
#pragma unroll
      for (int c = 0; c < kCols; ++c) {
        const int e = lane + 32 * c;
        if (e < d) {
          const float qv = qs[rr * (d + 1) + e], dyv = dys[rr * (d + 1) + e];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            adk[q][c] = fmaf(dss[(warp * 4 + q) * (kT + 1) + rr], qv, adk[q][c]);
            adv[q][c] = fmaf(ps[(warp * 4 + q) * (kT + 1) + rr], dyv, adv[q][c]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = t0 + warp * 4 + q;
    if (j >= a.N_C) continue;
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const int e = lane + 32 * c;
      if (e < d) {
        a.dk[(slot0 + j) * d + e] = adk[q][c] * a.rsd;
        a.dv[(slot0 + j) * d + e] = adv[q][c];
      }
    }
  }
}

template <int QT, int KV>
int run_bwd(const BwdArgs &a, int batch, cudaStream_t st) {
  const size_t smem = bwd_smem_bytes(a.d);
  for (auto fn : {bwd_rows_kernel<QT, KV>, bwd_slots_kernel<QT, KV>}) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(backward kernels) failed");
  }
  const int groups = batch * a.Hk;
  dim3 rg((a.q_g * a.S + kT - 1) / kT, groups);
  bwd_rows_kernel<QT, KV><<<rg, kBwdThreads, smem, st>>>(a);
  int rc = check_launch("bwd_rows_kernel");
  if (rc) return rc;
  dim3 sg((a.N_C + kT - 1) / kT, groups);
  bwd_slots_kernel<QT, KV><<<sg, kBwdThreads, smem, st>>>(a);
  return check_launch("bwd_slots_kernel");
}

}  // namespace

int launch_attn_backward(h2okv_cache *c, const void *q, const void *dy, const float *lse, int S,
                         int64_t P, float *dq, float *dk, float *dv, cudaStream_t st) {
  const h2okv_cache_desc &d = c->desc;
  // bf16 cache, d = 128: the tensor-core kernels (attn_bwd_tc.cu)
  if (bwd_tc_supported(d)) return launch_attn_backward_tc(c, q, dy, lse, S, P, dq, dk, dv, st);
  BwdArgs a;
  a.q = q;
  a.dy = dy;
  a.lse = lse;
  a.keys = reinterpret_cast<const uint8_t *>(c->bufs.keys);
  a.values = reinterpret_cast<const uint8_t *>(c->bufs.values);
  a.k_scales = reinterpret_cast<const __half *>(c->bufs.k_scales);
  a.v_scales = reinterpret_cast<const __half *>(c->bufs.v_scales);
  a.token_pos = c->bufs.token_pos;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.D = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(c->bufs.workspace) + c->ws.lse2);
  a.Hq = d.n_q_heads;
  a.Hk = d.n_kv_heads;
  a.q_g = d.n_q_heads / d.n_kv_heads;
  a.d = d.head_dim;
  a.N_C = d.capacity;
  a.S = S;
  a.P = (int)P;
  a.row_bytes = c->row_bytes;
  a.c2 = (float)(1.4426950408889634 / sqrt((double)d.head_dim));
  a.rsd = (float)(1.0 / sqrt((double)d.head_dim));
  if (d.q_dtype == H2OKV_F32) return run_bwd<H2OKV_F32, H2OKV_F32>(a, d.batch, st);
  switch (d.kv_dtype) {
    case H2OKV_BF16: return run_bwd<H2OKV_BF16, H2OKV_BF16>(a, d.batch, st);
    case H2OKV_I8: return run_bwd<H2OKV_BF16, H2OKV_I8>(a, d.batch, st);
    case H2OKV_I4: return run_bwd<H2OKV_BF16, H2OKV_I4>(a, d.batch, st);
  }
  return set_error(H2OKV_ERR_UNSUPPORTED, "kv dtype");
}

}  // namespace h2okv
