// Gradients of a chunk's SDPA over a bf16 cache with d = 128 on the tensor cores
// ("Learning how to Forget", §A.5: autograd runs over each chunk's computation while
// the cache decisions are replayed).  For query head h of group g, row i (token P + i)
// and slot j, with p_ij = exp(q_i.k_j / sqrt(d) - lse_i) on the visible slots
// (P + i >= t_j), dP_ij = dy_i.v_j, D_i = sum_j p_ij dP_ij, dS_ij = p_ij (dP_ij - D_i):
//   dq_i = sum_j dS_ij k_j / sqrt(d),
//   dk_j = sum over the group's heads and rows of dS_ij q_i / sqrt(d),
//   dv_j = sum over the group's heads and rows of p_ij dy_i.
// Two kernels, each with one loader warp (TMA, no multicast), one MMA warp and one
// warpgroup whose threads own the 128 TMEM lanes:
//   bwd_dq_tc_kernel    one CTA per 128 packed rows of a group (row-stationary):
//                       streams the group's K/V tiles twice.  Pass 1: S = Q K^T and
//                       dP = dY V^T into TMEM, D_i summed in registers (one thread per
//                       row).  Pass 2: S, dP again; dS written to TMEM (hi term over
//                       S, lo term in spare columns); dQ += dS K with dS read from
//                       TMEM.  Writes dq and D.
//   bwd_dkdv_tc_kernel  one CTA per 128 slots of a group (slot-stationary): streams
//                       every packed row tile of the group.  S^T = K Q^T and
//                       dP^T = V dY^T into TMEM; one thread per slot forms P^T and dS^T
//                       (written back over S^T / dP^T as hi and lo terms); dV += P^T dY
//                       and dK += dS^T Q with P^T, dS^T read from TMEM.
// Every output element is summed by one CTA in a fixed order (no atomics).  The
// probabilities and dS enter the second products as two bf16 terms each (hi + lo,
// one MMA per term): a single bf16 rounding of dS, amplified by the cancellation in
// the sums over slots and rows, would cost about 3e-3 of the largest gradient.
// Every wait is bounded; a timeout sets the cache's device status word and the CTA
// drains its MMAs before freeing TMEM.
#include "h2okv_internal.cuh"
#include "tc_ptx.cuh"

namespace h2okv {
namespace {

using namespace ptx;

constexpr int BT = 128;                      // rows / slots per tile
constexpr int HD = 128;                      // head dim
constexpr uint32_t kTile = BT * HD * 2;      // one bf16 tile: two 64-column swizzled halves
constexpr uint32_t kHalf = kTile / 2;
constexpr int kThr = 192;                    // warp 0 loads, warp 1 MMAs, warps 2-5 lanes
constexpr float kFar = 1048576.f;            // relative position no row of the chunk reaches
constexpr uint32_t IDESC_KK = idesc_bf16_f32(128, 128, false, false);  // A, B K-major
constexpr uint32_t IDESC_TM = idesc_bf16_f32(128, 128, false, true);   // A (TMEM), B MN-major

// K-major SW128 operand (128 rows x 128 columns): k-step ks covers 16 columns.
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int ks) {
  return desc_sw128(base + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
}
// The same tile as an MN-major operand (K = its rows): k-step ks covers 16 rows.
__device__ __forceinline__ uint64_t mdesc(uint32_t base, int ks) {
  return desc_sw128(base + ks * 2048, kHalf, 1024);
}
// Two values as bf16 pairs split in two terms: x = hi + lo up to 2^-17 |x|
// (hi = bf16(x), lo = bf16(x - hi)); the products that take them run once per term.
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

struct BwdTcParams {
  const int32_t *token_pos;  // [B*Hk][N_C]
  const float *lse;          // [B*Hq][S] natural-log row log-sum-exp of the forward
  float *D;                  // [B*Hq][S] (written by the dq kernel, read by the dk/dv kernel)
  float *dq, *dk, *dv;
  int *status;
  int Hq, Hk, q_g, N_C, S, P, tiles, n_kt;
  float c2, rsd;             // log2(e) / sqrt(d), 1 / sqrt(d)
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void fail(const BwdTcParams &p, bool &aborted) {
  if (!aborted) atomicExch(p.status, H2OKV_ERR_TIMEOUT);
  aborted = true;
}
// all 32 lanes wait; the result is warp-uniform
__device__ __forceinline__ bool wwait(uint64_t *bar, uint32_t parity, uint64_t lim) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, lim));
}
__device__ __forceinline__ float rel_of(const int32_t *tpg, int j, int N_C, int P) {
  if (j >= N_C) return kFar;
  const int64_t r = (int64_t)tpg[j] - (int64_t)P;
  return (float)(r < -1 ? -1 : (r > (int64_t)kFar ? (int64_t)kFar : r));
}

// ---- dq (and D) ----------------------------------------------------------------------
constexpr uint32_t Q_OFF = 0, DY_OFF = kTile, K_OFF = 2 * kTile, V_OFF = 4 * kTile;
constexpr uint32_t REL_OFF = 6 * kTile;                    // float [2 stages][BT]
constexpr uint32_t QBAR_OFF = REL_OFF + 2 * BT * 4;
enum { QB_Q = 0, QB_KF0, QB_KE0 = QB_KF0 + 2, QB_SF = QB_KE0 + 2, QB_SR, QB_PF, QB_DONE, QB_END };
constexpr uint32_t QTMEM_OFF = QBAR_OFF + QB_END * 8;
constexpr uint32_t kSmemDq = QTMEM_OFF + 16;
static_assert(kSmemDq + 1024 <= 232448, "dq shared memory budget");

__global__ void __launch_bounds__(kThr, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap q_map,
                     const __grid_constant__ CUtensorMap dy_map,
                     const __grid_constant__ CUtensorMap k_map,
                     const __grid_constant__ CUtensorMap v_map, const BwdTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled tiles need a 1024-byte aligned base
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  float *rel_s = reinterpret_cast<float *>(smem + REL_OFF);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + QBAR_OFF);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + QTMEM_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rt = p.q_g * p.tiles;
  const int bg = blockIdx.x / n_rt, rt = blockIdx.x % n_rt;
  const int b = bg / p.Hk, g = bg % p.Hk;
  const int hl = rt / p.tiles, t = rt % p.tiles;
  const int bhq = b * p.Hq + g * p.q_g + hl, i0 = t * BT;
  const int n_kt = p.n_kt, n_it = 2 * n_kt;  // K/V tiles streamed: pass 1, then pass 2
  const uint64_t lim = p.timeout_ns;
  if (threadIdx.x == 0) {
    mbar_init(&bar[QB_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[QB_KF0 + s], 1);
      mbar_init(&bar[QB_KE0 + s], 1 + 4);  // MMA commit + the lane warps (slot positions)
    }
    mbar_init(&bar[QB_SF], 1);
    mbar_init(&bar[QB_SR], 4);
    mbar_init(&bar[QB_PF], 4);
    mbar_init(&bar[QB_DONE], 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_s, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_s;
  bool aborted = false;

  if (warp == 0) {
    // ------------------------------------------ loads: Q, dY once; K, V, positions per tile
    const int32_t *tpg = p.token_pos + (size_t)bg * p.N_C;
    if (lane == 0) {
      mbar_expect_tx(&bar[QB_Q], 2 * kTile);
      tma_load_3d(smem + Q_OFF, &q_map, &bar[QB_Q], 0, i0, bhq);
      tma_load_3d(smem + Q_OFF + kHalf, &q_map, &bar[QB_Q], 64, i0, bhq);
      tma_load_3d(smem + DY_OFF, &dy_map, &bar[QB_Q], 0, i0, bhq);
      tma_load_3d(smem + DY_OFF + kHalf, &dy_map, &bar[QB_Q], 64, i0, bhq);
      mbar_arrive(&bar[QB_Q]);
    }
    int it = 0;
    for (; it < n_it && !aborted; ++it) {
      const int s = it & 1, use = it >> 1, kt = it % n_kt;
      if (use > 0 && !wwait(&bar[QB_KE0 + s], (use - 1) & 1, lim)) { fail(p, aborted); break; }
      for (int e = lane; e < BT; e += 32) rel_s[s * BT + e] = rel_of(tpg, kt * BT + e, p.N_C, p.P);
      __syncwarp();
      if (lane == 0) {
        mbar_expect_tx(&bar[QB_KF0 + s], 2 * kTile);
        tma_load_3d(smem + K_OFF + s * kTile, &k_map, &bar[QB_KF0 + s], 0, kt * BT, bg);
        tma_load_3d(smem + K_OFF + s * kTile + kHalf, &k_map, &bar[QB_KF0 + s], 64, kt * BT, bg);
        tma_load_3d(smem + V_OFF + s * kTile, &v_map, &bar[QB_KF0 + s], 0, kt * BT, bg);
        tma_load_3d(smem + V_OFF + s * kTile + kHalf, &v_map, &bar[QB_KF0 + s], 64, kt * BT, bg);
        mbar_arrive(&bar[QB_KF0 + s]);
      }
    }
    if (lane == 0) {  // the last loads land before exit
      mbar_wait(&bar[QB_Q], 0, 4000000000ull);
      for (int j = it - 1; j >= 0 && j >= it - 2; --j)
        mbar_wait(&bar[QB_KF0 + (j & 1)], (j >> 1) & 1, 4000000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = sbase + Q_OFF, dy_addr = sbase + DY_OFF;
      if (!mbar_wait(&bar[QB_Q], 0, lim)) fail(p, aborted);
      for (int it = 0; it < n_it && !aborted; ++it) {
        const int s = it & 1, use = it >> 1;
        const bool pass2 = it >= n_kt;
        if (!mbar_wait(&bar[QB_KF0 + s], use & 1, lim)) { fail(p, aborted); break; }
        // pass 1 holds no MMA behind the lanes' reads of S and dP: wait for them
        if (it > 0 && it - 1 < n_kt && !mbar_wait(&bar[QB_SR], (it - 1) & 1, lim)) {
          fail(p, aborted);
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = sbase + K_OFF + s * kTile, v_addr = sbase + V_OFF + s * kTile;
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks)
          mma_bf16_ss(tmem, kdesc(q_addr, ks), kdesc(k_addr, ks), IDESC_KK, ks > 0);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks)
          mma_bf16_ss(tmem + 128, kdesc(dy_addr, ks), kdesc(v_addr, ks), IDESC_KK, ks > 0);
        mma_commit(&bar[QB_SF]);
        if (pass2) {
          // dQ += dS K: dS over S in TMEM (two bf16 per column, 8 columns per k-step)
          if (!mbar_wait(&bar[QB_PF], (it - n_kt) & 1, lim)) { fail(p, aborted); break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < BT / 16; ++ks)
            mma_bf16_ts(tmem + 256, tmem + ks * 8, mdesc(k_addr, ks), IDESC_TM,
                        (it > n_kt || ks > 0) ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < BT / 16; ++ks)
            mma_bf16_ts(tmem + 256, tmem + 384 + ks * 8, mdesc(k_addr, ks), IDESC_TM, 1u);
        }
        mma_commit(&bar[QB_KE0 + s]);  // K, V of this stage no longer read
      }
      mma_commit(&bar[QB_DONE]);
      mbar_wait(&bar[QB_DONE], 0, 4000000000ull);  // drain before TMEM is freed
    }
    __syncwarp();
  } else {
    // ------------------------------------------------- one thread per row (TMEM lane)
    const int quarter = warp & 3;
    const int r = 32 * quarter + lane;
    const uint32_t lb = (uint32_t)(32 * quarter) << 16;
    const bool row_ok = i0 + r < p.S;
    float lse2 = row_ok ? p.lse[(size_t)bhq * p.S + i0 + r] * 1.4426950408889634f : INFINITY;
    if (!(lse2 > -INFINITY && lse2 < INFINITY)) lse2 = INFINITY;  // sees nothing / past the chunk: p = 0
    const float ri = (float)(i0 + r), c2 = p.c2;
    float Dacc = 0.f;
    for (int it = 0; it < n_it && !aborted; ++it) {
      const int s = it & 1, use = it >> 1;
      const bool pass2 = it >= n_kt;
      if (!wwait(&bar[QB_SF], it & 1, lim)) { fail(p, aborted); break; }
      if (!wwait(&bar[QB_KF0 + s], use & 1, lim)) { fail(p, aborted); break; }
      tc_fence_after();
      const float *rel = rel_s + s * BT;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t sv[64], dp[64];
        tmem_ld32(tmem + lb + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(sv));
        tmem_ld32(tmem + lb + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
        tmem_ld32(tmem + lb + 128 + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(dp));
        tmem_ld32(tmem + lb + 128 + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(dp + 32));
        tmem_wait_ld();
        if (!pass2) {
#pragma unroll
          for (int e = 0; e < 64; ++e) {
            const float pe = rel[64 * h + e] <= ri ? ex2(__uint_as_float(sv[e]) * c2 - lse2) : 0.f;
            Dacc = fmaf(pe, __uint_as_float(dp[e]), Dacc);
          }
        } else {
          uint32_t hi[32], lo[32];
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float p0 = rel[64 * h + e] <= ri ? ex2(__uint_as_float(sv[e]) * c2 - lse2) : 0.f;
            const float p1 =
                rel[64 * h + e + 1] <= ri ? ex2(__uint_as_float(sv[e + 1]) * c2 - lse2) : 0.f;
            split2(p0 * (__uint_as_float(dp[e]) - Dacc), p1 * (__uint_as_float(dp[e + 1]) - Dacc),
                   hi[e >> 1], lo[e >> 1]);
          }
          // dS of slots 64h .. 64h + 63: hi into columns 32h .. 32h + 31 (S there is
          // read), lo into 384 + 32h ..
          tmem_st32(tmem + lb + 32 * h, hi);
          tmem_st32(tmem + lb + 384 + 32 * h, lo);
        }
      }
      if (pass2) tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[pass2 ? QB_PF : QB_SR]);
        mbar_arrive(&bar[QB_KE0 + s]);  // slot positions no longer read
      }
      if (it == n_kt - 1 && row_ok) p.D[(size_t)bhq * p.S + i0 + r] = Dacc;
    }
    if (!aborted && wwait(&bar[QB_DONE], 0, lim)) {
      tc_fence_after();
      float *dst = p.dq + ((size_t)bhq * p.S + i0 + r) * HD;
#pragma unroll 1
      for (int cq = 0; cq < 4; ++cq) {
        uint32_t o[32];
        tmem_ld32(tmem + lb + 256 + 32 * cq, o);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4 *>(dst + 32 * cq)[e] =
                make_float4(__uint_as_float(o[4 * e]) * p.rsd, __uint_as_float(o[4 * e + 1]) * p.rsd,
                            __uint_as_float(o[4 * e + 2]) * p.rsd, __uint_as_float(o[4 * e + 3]) * p.rsd);
        }
      }
    } else if (!aborted) {
      fail(p, aborted);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- dk, dv --------------------------------------------------------------------------
constexpr uint32_t KK_OFF = 0, KV_OFF = kTile, KQ_OFF = 2 * kTile, KDY_OFF = 4 * kTile;
constexpr uint32_t ROWS_OFF = 6 * kTile;                     // float [2 stages][2][BT]: lse2, D
constexpr uint32_t KBAR_OFF = ROWS_OFF + 2 * 2 * BT * 4;
enum { KB_KV = 0, KB_QF0, KB_QE0 = KB_QF0 + 2, KB_SF = KB_QE0 + 2, KB_PF, KB_DONE, KB_END };
constexpr uint32_t KTMEM_OFF = KBAR_OFF + KB_END * 8;
constexpr uint32_t kSmemKv = KTMEM_OFF + 16;
static_assert(kSmemKv + 1024 <= 232448, "dk/dv shared memory budget");

__global__ void __launch_bounds__(kThr, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap q_map,
                       const __grid_constant__ CUtensorMap dy_map,
                       const __grid_constant__ CUtensorMap k_map,
                       const __grid_constant__ CUtensorMap v_map, const BwdTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  float *rows_s = reinterpret_cast<float *>(smem + ROWS_OFF);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + KBAR_OFF);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + KTMEM_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = blockIdx.x / p.n_kt, kt = blockIdx.x % p.n_kt;
  const int b = bg / p.Hk, g = bg % p.Hk;
  const int n_rt = p.q_g * p.tiles;
  const uint64_t lim = p.timeout_ns;
  if (threadIdx.x == 0) {
    mbar_init(&bar[KB_KV], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[KB_QF0 + s], 1);
      mbar_init(&bar[KB_QE0 + s], 1 + 4);  // MMA commit + the lane warps (lse2, D)
    }
    mbar_init(&bar[KB_SF], 1);
    mbar_init(&bar[KB_PF], 4);
    mbar_init(&bar[KB_DONE], 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_s, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_s;
  bool aborted = false;

  if (warp == 0) {
    // --------------------------- loads: K, V once; Q, dY, lse2 and D per packed row tile
    if (lane == 0) {
      mbar_expect_tx(&bar[KB_KV], 2 * kTile);
      tma_load_3d(smem + KK_OFF, &k_map, &bar[KB_KV], 0, kt * BT, bg);
      tma_load_3d(smem + KK_OFF + kHalf, &k_map, &bar[KB_KV], 64, kt * BT, bg);
      tma_load_3d(smem + KV_OFF, &v_map, &bar[KB_KV], 0, kt * BT, bg);
      tma_load_3d(smem + KV_OFF + kHalf, &v_map, &bar[KB_KV], 64, kt * BT, bg);
      mbar_arrive(&bar[KB_KV]);
    }
    int it = 0;
    for (; it < n_rt && !aborted; ++it) {
      const int s = it & 1, use = it >> 1;
      const int hl = it / p.tiles, t = it % p.tiles;
      const int bhq = b * p.Hq + g * p.q_g + hl, i0 = t * BT;
      if (use > 0 && !wwait(&bar[KB_QE0 + s], (use - 1) & 1, lim)) { fail(p, aborted); break; }
      for (int r = lane; r < BT; r += 32) {
        const bool ok = i0 + r < p.S;
        float l2 = ok ? p.lse[(size_t)bhq * p.S + i0 + r] * 1.4426950408889634f : INFINITY;
        if (!(l2 > -INFINITY && l2 < INFINITY)) l2 = INFINITY;  // sees nothing / past the chunk: p = 0
        rows_s[(s * 2 + 0) * BT + r] = l2;
        rows_s[(s * 2 + 1) * BT + r] = ok ? p.D[(size_t)bhq * p.S + i0 + r] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_expect_tx(&bar[KB_QF0 + s], 2 * kTile);
        tma_load_3d(smem + KQ_OFF + s * kTile, &q_map, &bar[KB_QF0 + s], 0, i0, bhq);
        tma_load_3d(smem + KQ_OFF + s * kTile + kHalf, &q_map, &bar[KB_QF0 + s], 64, i0, bhq);
        tma_load_3d(smem + KDY_OFF + s * kTile, &dy_map, &bar[KB_QF0 + s], 0, i0, bhq);
        tma_load_3d(smem + KDY_OFF + s * kTile + kHalf, &dy_map, &bar[KB_QF0 + s], 64, i0, bhq);
        mbar_arrive(&bar[KB_QF0 + s]);
      }
    }
    if (lane == 0) {
      mbar_wait(&bar[KB_KV], 0, 4000000000ull);
      for (int j = it - 1; j >= 0 && j >= it - 2; --j)
        mbar_wait(&bar[KB_QF0 + (j & 1)], (j >> 1) & 1, 4000000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t k_addr = sbase + KK_OFF, v_addr = sbase + KV_OFF;
      if (!mbar_wait(&bar[KB_KV], 0, lim)) fail(p, aborted);
      for (int it = 0; it < n_rt && !aborted; ++it) {
        const int s = it & 1, use = it >> 1;
        if (!mbar_wait(&bar[KB_QF0 + s], use & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        const uint32_t q_addr = sbase + KQ_OFF + s * kTile, dy_addr = sbase + KDY_OFF + s * kTile;
        // S^T = K Q^T, dP^T = V dY^T (slots on lanes).  The previous tile's dV / dK products
        // read P^T and dS^T from these columns first: one thread's MMAs run in order.
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks)
          mma_bf16_ss(tmem, kdesc(k_addr, ks), kdesc(q_addr, ks), IDESC_KK, ks > 0);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks)
          mma_bf16_ss(tmem + 128, kdesc(v_addr, ks), kdesc(dy_addr, ks), IDESC_KK, ks > 0);
        mma_commit(&bar[KB_SF]);
        if (!mbar_wait(&bar[KB_PF], it & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        // dV += P^T dY, dK += dS^T Q (A from TMEM: hi terms at 0 / 128, lo terms at
        // 64 / 192; B: the row tiles as MN-major operands)
#pragma unroll
        for (int ks = 0; ks < BT / 16; ++ks)
          mma_bf16_ts(tmem + 256, tmem + ks * 8, mdesc(dy_addr, ks), IDESC_TM,
                      (it > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < BT / 16; ++ks)
          mma_bf16_ts(tmem + 256, tmem + 64 + ks * 8, mdesc(dy_addr, ks), IDESC_TM, 1u);
#pragma unroll
        for (int ks = 0; ks < BT / 16; ++ks)
          mma_bf16_ts(tmem + 384, tmem + 128 + ks * 8, mdesc(q_addr, ks), IDESC_TM,
                      (it > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < BT / 16; ++ks)
          mma_bf16_ts(tmem + 384, tmem + 192 + ks * 8, mdesc(q_addr, ks), IDESC_TM, 1u);
        mma_commit(&bar[KB_QE0 + s]);  // Q, dY of this stage no longer read
      }
      mma_commit(&bar[KB_DONE]);
      mbar_wait(&bar[KB_DONE], 0, 4000000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ one thread per slot (TMEM lane)
    const int quarter = warp & 3;
    const int jl = 32 * quarter + lane;
    const int j = kt * BT + jl;
    const uint32_t lb = (uint32_t)(32 * quarter) << 16;
    const float rel = rel_of(p.token_pos + (size_t)bg * p.N_C, j, p.N_C, p.P);
    const float c2 = p.c2;
    for (int it = 0; it < n_rt && !aborted; ++it) {
      const int s = it & 1, use = it >> 1;
      const int t = it % p.tiles, i0 = t * BT;
      if (!wwait(&bar[KB_SF], it & 1, lim)) { fail(p, aborted); break; }
      if (!wwait(&bar[KB_QF0 + s], use & 1, lim)) { fail(p, aborted); break; }
      tc_fence_after();
      // row r of the tile sees this slot iff i0 + r >= rel; rows past the chunk have
      // lse2 = +inf
      const float rmin = rel - (float)i0;
      const float *l2 = rows_s + (s * 2 + 0) * BT, *Dr = rows_s + (s * 2 + 1) * BT;
      // by quarters of 32 rows (S^T columns 32q .. 32q + 31): hi terms of P^T into
      // columns 16q .., of dS^T into 128 + 16q .. (all read already); lo terms into
      // 64 + 16q .. and 192 + 16q .., written once quarter 2 (for q = 0, 1) or 3 (for
      // q = 2, 3) has read those columns
      uint32_t plo[4][16], dlo[4][16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t sv[32], dp[32], phi[16], dhi[16];
        tmem_ld32(tmem + lb + 32 * q, sv);
        tmem_ld32(tmem + lb + 128 + 32 * q, dp);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int r = 32 * q + e;
          const float p0 = (float)r >= rmin ? ex2(__uint_as_float(sv[e]) * c2 - l2[r]) : 0.f;
          const float p1 = (float)(r + 1) >= rmin ? ex2(__uint_as_float(sv[e + 1]) * c2 - l2[r + 1]) : 0.f;
          split2(p0, p1, phi[e >> 1], plo[q][e >> 1]);
          split2(p0 * (__uint_as_float(dp[e]) - Dr[r]), p1 * (__uint_as_float(dp[e + 1]) - Dr[r + 1]),
                 dhi[e >> 1], dlo[q][e >> 1]);
        }
        tmem_st16(tmem + lb + 16 * q, phi);
        tmem_st16(tmem + lb + 128 + 16 * q, dhi);
        if (q >= 2) {
#pragma unroll
          for (int u = 2 * (q - 2); u < 2 * (q - 2) + 2; ++u) {
            tmem_st16(tmem + lb + 64 + 16 * u, plo[u]);
            tmem_st16(tmem + lb + 192 + 16 * u, dlo[u]);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[KB_PF]);
        mbar_arrive(&bar[KB_QE0 + s]);  // lse2, D of this stage no longer read
      }
    }
    if (!aborted && wwait(&bar[KB_DONE], 0, lim)) {
      tc_fence_after();
      const bool ok = j < p.N_C;
      float *dvr = p.dv + ((size_t)bg * p.N_C + j) * HD;
      float *dkr = p.dk + ((size_t)bg * p.N_C + j) * HD;
#pragma unroll 1
      for (int cq = 0; cq < 8; ++cq) {
        uint32_t o[32];
        tmem_ld32(tmem + lb + 256 + 32 * cq, o);  // dV (cq < 4), then dK
        tmem_wait_ld();
        if (ok) {
          float *dst = cq < 4 ? dvr + 32 * cq : dkr + 32 * (cq - 4);
          const float f = cq < 4 ? 1.f : p.rsd;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4 *>(dst)[e] =
                make_float4(__uint_as_float(o[4 * e]) * f, __uint_as_float(o[4 * e + 1]) * f,
                            __uint_as_float(o[4 * e + 2]) * f, __uint_as_float(o[4 * e + 3]) * f);
        }
      }
    } else if (!aborted) {
      fail(p, aborted);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <typename K>
int opt_in(K kernel, uint32_t smem, bool &done) {
  if (done) return H2OKV_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(backward tensor-core kernels) failed");
  done = true;
  return H2OKV_OK;
}

}  // namespace

bool bwd_tc_supported(const h2okv_cache_desc &d) {
  return d.head_dim == HD && d.q_dtype == H2OKV_BF16 && d.kv_dtype == H2OKV_BF16;
}

int launch_attn_backward_tc(h2okv_cache *c, const void *q, const void *dy, const float *lse, int S,
                            int64_t P, float *dq, float *dk, float *dv, cudaStream_t st) {
  const h2okv_cache_desc &d = c->desc;
  int rc = ensure_cache_maps(c);
  if (rc) return rc;
  CUtensorMap qmap, dymap;
  rc = encode_rows_map(&qmap, q, (uint64_t)S, (uint64_t)d.batch * d.n_q_heads);
  if (rc) return rc;
  rc = encode_rows_map(&dymap, dy, (uint64_t)S, (uint64_t)d.batch * d.n_q_heads);
  if (rc) return rc;
  BwdTcParams p;
  uint8_t *ws = reinterpret_cast<uint8_t *>(c->bufs.workspace);
  p.token_pos = c->bufs.token_pos;
  p.lse = lse;
  p.D = reinterpret_cast<float *>(ws + c->ws.lse2);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.status = reinterpret_cast<int *>(ws + c->ws.status);
  p.Hq = d.n_q_heads;
  p.Hk = d.n_kv_heads;
  p.q_g = d.n_q_heads / d.n_kv_heads;
  p.N_C = d.capacity;
  p.S = S;
  p.P = (int)P;
  p.tiles = (S + BT - 1) / BT;
  p.n_kt = (d.capacity + BT - 1) / BT;
  p.c2 = (float)(1.4426950408889634 / 11.313708498984761);  // log2(e) / sqrt(128)
  p.rsd = (float)(1.0 / 11.313708498984761);
  p.timeout_ns = c->wait_timeout_ns;
  static thread_local int ready_dev = -1;
  static thread_local bool done_q = false, done_kv = false;
  int dev = 0;
  cudaGetDevice(&dev);
  if (ready_dev != dev) {
    done_q = done_kv = false;
    ready_dev = dev;
  }
  rc = opt_in(bwd_dq_tc_kernel, kSmemDq + 1024, done_q);
  if (rc) return rc;
  rc = opt_in(bwd_dkdv_tc_kernel, kSmemKv + 1024, done_kv);
  if (rc) return rc;
  const CUtensorMap &kmap = *reinterpret_cast<const CUtensorMap *>(c->tc.k_map);
  const CUtensorMap &vmap = *reinterpret_cast<const CUtensorMap *>(c->tc.v_map);
  const long long groups = (long long)d.batch * d.n_kv_heads;
  const long long g_dq = groups * p.q_g * p.tiles, g_kv = groups * p.n_kt;
  if (g_dq > INT32_MAX || g_kv > INT32_MAX)
    return set_error(H2OKV_ERR_UNSUPPORTED, "backward grid too large");
  bwd_dq_tc_kernel<<<(unsigned)g_dq, kThr, kSmemDq + 1024, st>>>(qmap, dymap, kmap, vmap, p);
  rc = check_launch("bwd_dq_tc_kernel");
  if (rc) return rc;
  bwd_dkdv_tc_kernel<<<(unsigned)g_kv, kThr, kSmemKv + 1024, st>>>(qmap, dymap, kmap, vmap, p);
  return check_launch("bwd_dkdv_tc_kernel");
}

}  // namespace h2okv
