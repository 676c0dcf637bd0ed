// Tensor-core path of chunked cache attention with summed weights for d = 128
// and a bf16 cache ("Learning how to Forget", §A.1 token-position mask, §A.7
// SDPA plus the attention weights summed over the query axis, returned per KV
// slot and summed over the q_g query heads of each GQA group).
//
// One CTA owns 128 query rows of one head (rows past S are zero-filled by TMA
// and never written).  It streams the head's KV group twice:
//
//   phase A  S = Q K^T per 128-slot tile (tcgen05.mma, M=128 rows, N=128 slots,
//            K=128, accumulator in TMEM); one softmax thread per row reads its
//            row with tcgen05.ld and keeps the online max / sum -> base-2 LSE.
//   phase B  S^T = K Q^T per tile (M=128 slots, N=128 rows): one thread per
//            SLOT reads its 128 logits, forms p = exp2(s*log2e/sqrt(d) - lse2_i)
//            with the FINAL row LSE, sums them in registers (the slot's summed
//            weight over this CTA's rows: no atomics, deterministic) and writes
//            p as bf16 into shared memory (MN-major operand layout); then
//            O += P V (tcgen05.mma, A = P MN-major, B = V MN-major) in TMEM.
//            P is already normalised, so O needs no rescaling.
//
// Warp roles (256 threads): warp 0 TMA producer (K/V tiles via
// cp.async.bulk.tensor, no multicast; token positions via plain loads), warp 1
// TMEM allocator and single-thread MMA issuer, warps 4-7 softmax / column sums /
// epilogue (warp 4+q owns TMEM lanes 32q..32q+31).  Two K/V stages and two TMEM
// S buffers let the MMA of tile kt+1 overlap the softmax of tile kt.  Every
// wait is bounded; a timeout sets the cache's device status word and the CTA
// drains its copies and MMAs before freeing TMEM.
//
// Per-(row tile, slot) sums go to a partial buffer; a small reduction kernel
// sums them in a fixed order into w [B, H_k, N_C] and wq [B, H_q, N_C].
#include <stdio.h>

#include "h2okv_internal.cuh"
#include "tc_ptx.cuh"

namespace h2okv {
namespace {

using namespace ptx;

constexpr int BM = 128;        // query rows per CTA
constexpr int BN = 128;        // slots per tile
constexpr int D = 128;         // head dim
constexpr int kThreads = 256;
constexpr uint32_t kTileBytes = BM * D * 2;  // 32 KiB (two 64-column swizzled halves)
constexpr uint32_t kHalfBytes = kTileBytes / 2;

// shared memory carve-up (offsets from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K0 = OFF_Q + kTileBytes;
constexpr uint32_t OFF_V0 = OFF_K0 + kTileBytes;
constexpr uint32_t OFF_K1 = OFF_V0 + kTileBytes;
constexpr uint32_t OFF_V1 = OFF_K1 + kTileBytes;
constexpr uint32_t OFF_P0 = OFF_V1 + kTileBytes;
constexpr uint32_t OFF_P1 = OFF_P0 + kTileBytes;
constexpr uint32_t OFF_TP = OFF_P1 + kTileBytes;       // int32 [2][BN]
constexpr uint32_t OFF_TPMAX = OFF_TP + 2 * BN * 4;    // int32 [2] (+pad)
constexpr uint32_t OFF_LSE = OFF_TPMAX + 16;           // float [BM]
constexpr uint32_t OFF_BAR = OFF_LSE + BM * 4;         // uint64 barriers
constexpr int NBAR = 15;
constexpr uint32_t OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr uint32_t kSmemBytes = OFF_TMEM + 16 + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;  // S buffers at 0 and 128, O at 256
constexpr uint32_t IDESC_K_MAJOR = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, true, true);

struct TcParams {
  const int32_t *token_pos;  // [B*Hk][N_C]
  __nv_bfloat16 *y;          // [B*Hq][S][D]
  float *lse_out;            // [B*Hq][S] or null
  float *part_w;             // [B*Hq*tiles][N_C]
  int *status;               // device status word (0 = ok)
  int Hq, Hk, q_g, N_C, S, P, tiles, n_kt;
  float scale2;  // log2(e) / sqrt(d)
  unsigned long long timeout_ns;
};

enum { B_Q = 0, B_FULL0, B_FULL1, B_EMPTY0, B_EMPTY1, B_SFULL0, B_SFULL1, B_SFREE0, B_SFREE1,
       B_PFULL0, B_PFULL1, B_PFREE0, B_PFREE1, B_OFULL, B_DRAIN };

// K-major SW128 operand (rows x 128 columns as two 64-column halves): k-step ks
// (16 columns) starts 32 bytes further inside a half.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int ks) {
  return desc_sw128(base + (ks >> 2) * kHalfBytes + (ks & 3) * 32, 16, 1024);
}
// MN-major SW128 operand (two 64-element MN blocks 16 KiB apart, K rows of 128 B,
// 8 K rows per 1024 B atom): k-step ks covers 16 K rows.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int ks) {
  return desc_sw128(base + ks * 2048, kHalfBytes, 1024);
}

// All 32 lanes wait; the result is made warp-uniform so that a timeout seen by
// one lane never splits the warp before a .sync.aligned instruction.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, uint64_t lim) {
  const bool ok = mbar_wait(bar, parity, lim);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void fail(const TcParams &p, bool &aborted) {
  if (!aborted) atomicExch(p.status, H2OKV_ERR_TIMEOUT);
  aborted = true;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap q_map,
                   const __grid_constant__ CUtensorMap k_map,
                   const __grid_constant__ CUtensorMap v_map, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  int32_t *tp_s = reinterpret_cast<int32_t *>(smem + OFF_TP);
  int32_t *tpmax_s = reinterpret_cast<int32_t *>(smem + OFF_TPMAX);
  float *lse_s = reinterpret_cast<float *>(smem + OFF_LSE);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + OFF_TMEM);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w = blockIdx.x;
  const int bhq = w / p.tiles, t = w - bhq * p.tiles;
  const int b = bhq / p.Hq, h = bhq - b * p.Hq;
  const int bg = b * p.Hk + h / p.q_g;
  const int i0 = t * BM;
  const int n_kt = p.n_kt;
  const uint64_t lim = p.timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(&bar[B_Q], 1);
    mbar_init(&bar[B_FULL0], 1);
    mbar_init(&bar[B_FULL1], 1);
    mbar_init(&bar[B_EMPTY0], 5);  // MMA commit + 4 softmax warps
    mbar_init(&bar[B_EMPTY1], 5);
    mbar_init(&bar[B_SFULL0], 1);
    mbar_init(&bar[B_SFULL1], 1);
    mbar_init(&bar[B_SFREE0], 4);
    mbar_init(&bar[B_SFREE1], 4);
    mbar_init(&bar[B_PFULL0], 4);
    mbar_init(&bar[B_PFULL1], 4);
    mbar_init(&bar[B_PFREE0], 1);
    mbar_init(&bar[B_PFREE1], 1);
    mbar_init(&bar[B_OFULL], 1);
    mbar_init(&bar[B_DRAIN], 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_s, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&q_map);
    prefetch_tensormap(&k_map);
    prefetch_tensormap(&v_map);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_s;
  bool aborted = false;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(&bar[B_Q], kTileBytes);
      tma_load_3d(smem + OFF_Q, &q_map, &bar[B_Q], 0, i0, bhq);
      tma_load_3d(smem + OFF_Q + kHalfBytes, &q_map, &bar[B_Q], 64, i0, bhq);
      mbar_arrive(&bar[B_Q]);
    }
    const int32_t *tpg = p.token_pos + (size_t)bg * p.N_C;
    int issued = 0;
    for (int it = 0; it < 2 * n_kt && !aborted; ++it) {
      const bool phB = it >= n_kt;
      const int kt = phB ? it - n_kt : it;
      const int s = it & 1, n = it >> 1;
      if (n > 0 && !warp_wait(&bar[B_EMPTY0 + s], (n - 1) & 1, lim)) {
        fail(p, aborted);
        break;
      }
      uint8_t *kdst = smem + (s ? OFF_K1 : OFF_K0);
      uint8_t *vdst = smem + (s ? OFF_V1 : OFF_V0);
      if (lane == 0) {
        mbar_expect_tx(&bar[B_FULL0 + s], phB ? 2 * kTileBytes : kTileBytes);
        tma_load_3d(kdst, &k_map, &bar[B_FULL0 + s], 0, kt * BN, bg);
        tma_load_3d(kdst + kHalfBytes, &k_map, &bar[B_FULL0 + s], 64, kt * BN, bg);
        if (phB) {
          tma_load_3d(vdst, &v_map, &bar[B_FULL0 + s], 0, kt * BN, bg);
          tma_load_3d(vdst + kHalfBytes, &v_map, &bar[B_FULL0 + s], 64, kt * BN, bg);
        }
      }
      int32_t tmax = INT32_MIN;
#pragma unroll
      for (int e = lane; e < BN; e += 32) {
        const int j = kt * BN + e;
        const int32_t v = j < p.N_C ? tpg[j] : kEmptyPos;
        tp_s[s * BN + e] = v;
        tmax = max(tmax, v);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tmax = max(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
      if (lane == 0) tpmax_s[s] = tmax;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_FULL0 + s]);
      issued = it + 1;
    }
    // drain: the last (up to two) issued stage loads must land before exit
    if (lane == 0) {
      mbar_wait(&bar[B_Q], 0, 4000000000ull);
      for (int it = issued - 1; it >= 0 && it >= issued - 2; --it)
        mbar_wait(&bar[B_FULL0 + (it & 1)], (it >> 1) & 1, 4000000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = sbase + OFF_Q;
      if (!mbar_wait(&bar[B_Q], 0, lim)) fail(p, aborted);
      tc_fence_after();
      // phase A: S = Q K^T
      for (int kt = 0; kt < n_kt && !aborted; ++kt) {
        const int s = kt & 1, u = kt, buf = u & 1;
        if (!mbar_wait(&bar[B_FULL0 + s], (kt >> 1) & 1, lim)) { fail(p, aborted); break; }
        if (u >= 2 && !mbar_wait(&bar[B_SFREE0 + buf], ((u >> 1) - 1) & 1, lim)) {
          fail(p, aborted);
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = sbase + (s ? OFF_K1 : OFF_K0);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16_ss(tmem + buf * 128, kmajor_desc(q_addr, ks), kmajor_desc(k_addr, ks),
                      IDESC_K_MAJOR, ks > 0);
        mma_commit(&bar[B_SFULL0 + buf]);
        mma_commit(&bar[B_EMPTY0 + s]);
      }
      // phase B: S^T = K Q^T, then O += P V
      auto issue_st = [&](int kt) -> bool {
        const int it = n_kt + kt, s = it & 1, u = n_kt + kt, buf = u & 1;
        if (!mbar_wait(&bar[B_FULL0 + s], (it >> 1) & 1, lim)) return false;
        if (u >= 2 && !mbar_wait(&bar[B_SFREE0 + buf], ((u >> 1) - 1) & 1, lim)) return false;
        tc_fence_after();
        const uint32_t k_addr = sbase + (s ? OFF_K1 : OFF_K0);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16_ss(tmem + buf * 128, kmajor_desc(k_addr, ks), kmajor_desc(q_addr, ks),
                      IDESC_K_MAJOR, ks > 0);
        mma_commit(&bar[B_SFULL0 + buf]);
        return true;
      };
      if (!aborted && !issue_st(0)) fail(p, aborted);
      for (int kt = 0; kt < n_kt && !aborted; ++kt) {
        if (kt + 1 < n_kt && !issue_st(kt + 1)) { fail(p, aborted); break; }
        const int pb = kt & 1;
        if (!mbar_wait(&bar[B_PFULL0 + pb], (kt >> 1) & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        const int s = (n_kt + kt) & 1;
        const uint32_t v_addr = sbase + (s ? OFF_V1 : OFF_V0);
        const uint32_t p_addr = sbase + (pb ? OFF_P1 : OFF_P0);
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_bf16_ss(tmem + 256, mnmajor_desc(p_addr, ks), mnmajor_desc(v_addr, ks), IDESC_PV,
                      (kt > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bar[B_PFREE0 + pb]);
        mma_commit(&bar[B_EMPTY0 + s]);
      }
      mma_commit(&bar[B_OFULL]);
      // drain: every MMA issued by this thread completes before TMEM is freed
      mma_commit(&bar[B_DRAIN]);
      mbar_wait(&bar[B_DRAIN], 0, 4000000000ull);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / sums
    const int st = threadIdx.x - 128;  // row (phase A) or slot (phase B) within the tile
    const uint32_t lane_base = (uint32_t)(32 * (warp - 4)) << 16;
    const float c2 = p.scale2;
    const int row_i = i0 + st;
    const int64_t row_lim = (int64_t)p.P + row_i;
    float m = -INFINITY, l = 0.f;
    uint32_t xr[BN];
    for (int kt = 0; kt < n_kt && !aborted; ++kt) {
      const int u = kt, buf = u & 1, s = kt & 1;
      if (!warp_wait(&bar[B_SFULL0 + buf], (u >> 1) & 1, lim)) { fail(p, aborted); break; }
      if (!warp_wait(&bar[B_FULL0 + s], (kt >> 1) & 1, lim)) { fail(p, aborted); break; }
      tc_fence_after();
      tmem_ld32(tmem + lane_base + buf * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(xr + 0));
      tmem_ld32(tmem + lane_base + buf * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(xr + 32));
      tmem_ld32(tmem + lane_base + buf * 128 + 64, *reinterpret_cast<uint32_t(*)[32]>(xr + 64));
      tmem_ld32(tmem + lane_base + buf * 128 + 96, *reinterpret_cast<uint32_t(*)[32]>(xr + 96));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_SFREE0 + buf]);
      const bool all_visible = (int64_t)tpmax_s[s] <= (int64_t)p.P + i0;
      if (!all_visible) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if ((int64_t)tp_s[s * BN + e] > row_lim) xr[e] = __float_as_uint(-INFINITY);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_EMPTY0 + s]);
      // row max with 8 independent chains
      float mx8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx8[q] = __uint_as_float(xr[q]);
#pragma unroll
      for (int e = 8; e < BN; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(xr[e]));
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_new = fmaxf(m, mx * c2);
      if (m_new == -INFINITY) continue;
      float sm8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) sm8[q] = 0.f;
#pragma unroll
      for (int e = 0; e < BN; ++e) sm8[e & 7] += ex2(fmaf(__uint_as_float(xr[e]), c2, -m_new));
      const float sum = ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) + ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]));
      l = l * ex2(m - m_new) + sum;
      m = m_new;
    }
    const float lse2 = (l > 0.f) ? m + lg2(l) : -INFINITY;
    lse_s[st] = lse2;
    if (p.lse_out && row_i < p.S) p.lse_out[(size_t)bhq * p.S + row_i] = lse2 * 0.69314718055994531f;
    named_bar_sync(1, 128);

    // phase B
    const int rmax = min(BM, p.S - i0);
    float *pw = p.part_w + ((size_t)bhq * p.tiles + t) * p.N_C;
    const uint32_t p_row = (st >> 3) * 1024 + (st & 7) * 128;
    uint32_t r[32];
    for (int kt = 0; kt < n_kt && !aborted; ++kt) {
      const int u = n_kt + kt, buf = u & 1, it = n_kt + kt, s = it & 1, pb = kt & 1;
      if (!warp_wait(&bar[B_SFULL0 + buf], (u >> 1) & 1, lim)) { fail(p, aborted); break; }
      if (!warp_wait(&bar[B_FULL0 + s], (it >> 1) & 1, lim)) { fail(p, aborted); break; }
      // P buffer pb was last read by the P V product of tile kt - 2
      if (kt >= 2 && !warp_wait(&bar[B_PFREE0 + pb], ((kt >> 1) - 1) & 1, lim)) {
        fail(p, aborted);
        break;
      }
      tc_fence_after();
      const int64_t tpj = tp_s[s * BN + st];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_EMPTY0 + s]);
      // visible rows r of this tile: tpj <= P + i0 + r, r < rmax
      const int64_t rm = tpj - (int64_t)p.P - i0;
      const int rmin = rm <= 0 ? 0 : (rm >= BM ? BM : (int)rm);
      const bool full = __all_sync(0xffffffffu, rmin == 0 && rmax == BM);
      const uint32_t p_buf = sbase + (pb ? OFF_P1 : OFF_P0) + p_row;
      float cs8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) cs8[q] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tmem + lane_base + buf * 128 + c * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int r0 = c * 32 + e;
          float p0 = ex2(fmaf(__uint_as_float(r[e]), c2, -lse_s[r0]));
          float p1 = ex2(fmaf(__uint_as_float(r[e + 1]), c2, -lse_s[r0 + 1]));
          if (!full) {
            p0 = (r0 >= rmin && r0 < rmax) ? p0 : 0.f;
            p1 = (r0 + 1 >= rmin && r0 + 1 < rmax) ? p1 : 0.f;
          }
          cs8[(e >> 1) & 7] += p0 + p1;
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
        // rows 32c .. 32c+31 = M block c/2, 16-byte chunks (c%2)*4 .. +3 of this slot's K row
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int cc = (c & 1) * 4 + q;
          const uint32_t addr = p_buf + (c >> 1) * kHalfBytes + ((cc ^ (st & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * q]),
                       "r"(pk[4 * q + 1]), "r"(pk[4 * q + 2]), "r"(pk[4 * q + 3])
                       : "memory");
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[B_SFREE0 + buf]);
        mbar_arrive(&bar[B_PFULL0 + pb]);
      }
      const float colsum = ((cs8[0] + cs8[1]) + (cs8[2] + cs8[3])) + ((cs8[4] + cs8[5]) + (cs8[6] + cs8[7]));
      const int j = kt * BN + st;
      if (j < p.N_C) pw[j] = colsum;
    }
    // epilogue: y = O (already normalised)
    if (!aborted && !warp_wait(&bar[B_OFULL], 0, lim)) fail(p, aborted);
    tc_fence_after();
    if (!aborted) {
      __nv_bfloat16 *yrow = p.y + ((size_t)bhq * p.S + row_i) * D;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tmem + lane_base + 256 + c * 32, r);
        tmem_wait_ld();
        if (row_i < p.S) {
          uint32_t o[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            o[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
          uint4 *dst = reinterpret_cast<uint4 *>(yrow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// w[b, g, j] = sum over the group's heads and row tiles of the partial sums;
// wq[b, h, j] = sum over the head's row tiles.  Fixed summation order.
__global__ void __launch_bounds__(256)
    reduce_w_kernel(const float *__restrict__ part_w, float *__restrict__ w,
                    float *__restrict__ wq, int Hq, int Hk, int q_g, int N_C, int tiles,
                    int tiles_used) {
  const int bg = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= N_C) return;
  const int b = bg / Hk, g = bg - b * Hk;
  float tot = 0.f;
  for (int hl = 0; hl < q_g; ++hl) {
    const int bhq = b * Hq + g * q_g + hl;
    const float *src = part_w + (size_t)bhq * tiles * N_C + j;
    float hs = 0.f;
    for (int t = 0; t < tiles_used; ++t) hs += src[(size_t)t * N_C];
    if (wq) wq[(size_t)bhq * N_C + j] = hs;
    tot += hs;
  }
  w[(size_t)bg * N_C + j] = tot;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D bf16 map over [planes][rows][128] with a (64 x 128 x 1) box, 128-byte swizzle.
int encode_rows_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t planes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(H2OKV_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)D, rows, planes};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(H2OKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return H2OKV_OK;
}

}  // namespace

bool tc_path_supported(const h2okv_cache_desc &d) {
  return d.head_dim == D && d.q_dtype == H2OKV_BF16 && d.kv_dtype == H2OKV_BF16;
}

void tc_plan(const h2okv_cache_desc &d, TcPlan *plan) {
  plan->enabled = tc_path_supported(d);
  plan->tiles_per_head = (d.max_chunk + BM - 1) / BM;
  plan->max_splits = 0;
}

int launch_attn_tc(h2okv_cache *c, const void *q, int S, int64_t P, void *y, float *lse, float *w,
                   float *wq, cudaStream_t st) {
  const h2okv_cache_desc &d = c->desc;
  uint8_t *ws = reinterpret_cast<uint8_t *>(c->bufs.workspace);
  if (!c->tc.maps_ready) {
    int rc = encode_rows_map(reinterpret_cast<CUtensorMap *>(c->tc.k_map), c->bufs.keys,
                             (uint64_t)d.capacity, (uint64_t)d.batch * d.n_kv_heads);
    if (rc) return rc;
    rc = encode_rows_map(reinterpret_cast<CUtensorMap *>(c->tc.v_map), c->bufs.values,
                         (uint64_t)d.capacity, (uint64_t)d.batch * d.n_kv_heads);
    if (rc) return rc;
    c->tc.maps_ready = true;
  }
  CUtensorMap qmap;
  int rc = encode_rows_map(&qmap, q, (uint64_t)S, (uint64_t)d.batch * d.n_q_heads);
  if (rc) return rc;

  static thread_local int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess)
      return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(attn_tc_kernel): %s",
                       cudaGetErrorString(e));
    configured_dev = dev;
  }
  TcParams prm;
  prm.token_pos = c->bufs.token_pos;
  prm.y = reinterpret_cast<__nv_bfloat16 *>(y);
  prm.lse_out = lse;
  prm.part_w = reinterpret_cast<float *>(ws + c->ws.part_w);
  prm.status = reinterpret_cast<int *>(ws + c->ws.status);
  prm.Hq = d.n_q_heads;
  prm.Hk = d.n_kv_heads;
  prm.q_g = d.n_q_heads / d.n_kv_heads;
  prm.N_C = d.capacity;
  prm.S = S;
  prm.P = (int)P;
  prm.tiles = (S + BM - 1) / BM;
  prm.n_kt = (d.capacity + BN - 1) / BN;
  prm.scale2 = (float)(1.4426950408889634 / 11.313708498984761);  // log2(e) / sqrt(128)
  prm.timeout_ns = c->wait_timeout_ns;
  const int grid = d.batch * d.n_q_heads * prm.tiles;
  attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(
      qmap, *reinterpret_cast<const CUtensorMap *>(c->tc.k_map),
      *reinterpret_cast<const CUtensorMap *>(c->tc.v_map), prm);
  rc = check_launch("attn_tc_kernel");
  if (rc) return rc;
  dim3 rgrid((d.capacity + 255) / 256, d.batch * d.n_kv_heads);
  reduce_w_kernel<<<rgrid, 256, 0, st>>>(prm.part_w, w, wq, d.n_q_heads, d.n_kv_heads, prm.q_g,
                                         d.capacity, prm.tiles, prm.tiles);
  return check_launch("reduce_w_kernel");
}

}  // namespace h2okv
