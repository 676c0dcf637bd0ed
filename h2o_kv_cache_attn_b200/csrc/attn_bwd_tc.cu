// Gradients of a chunk's SDPA over a bf16 cache with d = 128 on the tensor cores
// ("Learning how to Forget", §A.5: autograd runs over each chunk's computation while
// the cache decisions are replayed).  For query head h of group g, row i (token P + i)
// and slot j, with p_ij = exp(q_i.k_j / sqrt(d) - lse_i) on the visible slots
// (P + i >= t_j), dP_ij = dy_i.v_j, D_i = sum_j p_ij dP_ij, dS_ij = p_ij (dP_ij - D_i):
//   dq_i = sum_j dS_ij k_j / sqrt(d),
//   dk_j = sum over the group's heads and rows of dS_ij q_i / sqrt(d),
//   dv_j = sum over the group's heads and rows of p_ij dy_i.
// Three kernels, each with one loader warp (TMA, no multicast), one MMA warp and two
// warpgroups of lane warps (warps w and w + 4 share TMEM lane quarter w mod 4):
//   bwd_d_tc_kernel     one CTA per two 128-row tiles of a group's packed rows: S = Q K^T
//                       and dP = dY V^T of both tiles into TMEM per K/V tile (each K/V
//                       tile taken from L2 serves 256 rows); D_i = sum_j p_ij dP_ij in
//                       registers, one row per lane.
//   bwd_dq_tc_kernel    one CTA per 128 packed rows (row-stationary): per K/V tile S, dP
//                       (S double-buffered in TMEM), dS written back over S by 32-slot
//                       chunks (hi term, then lo term), dQ += dS K with dS read from
//                       TMEM, each chunk's products issued as soon as it is written; the
//                       two lane halves split the slots.  Writes dq.
//   bwd_dkdv_tc_kernel  one CTA per 128 slots of a group (slot-stationary): streams
//                       every packed row tile of the group.  S^T = K Q^T and
//                       dP^T = V dY^T into TMEM; one slot per lane forms P^T and dS^T
//                       by 32-row chunks (written back over S^T / dP^T as hi and lo
//                       terms); dV += P^T dY and dK += dS^T Q with P^T, dS^T read from
//                       TMEM, again chunk by chunk; the two lane halves split the rows.
// The dk/dv kernel is a programmatic dependent of the dq kernel: its CTAs take the SMs
// that the dq grid's last wave leaves idle.
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
constexpr int kLaneWarps = 8;                // two warps per TMEM lane quarter
constexpr int kThr = 64 + 32 * kLaneWarps;   // warp 0 loads, warp 1 MMAs, warps 2-9 lanes
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
__device__ __forceinline__ void split2(float2 x, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x.x, x.y);
  const float2 hf = __bfloat1622float2(h);
  const float2 d = fma2(hf, make_float2(-1.f, -1.f), x);
  const __nv_bfloat162 l = __floats2bfloat162_rn(d.x, d.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}
__device__ __forceinline__ float2 u2f2(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a), __uint_as_float(b));
}
__device__ __forceinline__ float2 ex2_2(float2 x) { return make_float2(ex2(x.x), ex2(x.y)); }

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

// Programmatic dependent launch: the dk/dv kernel may be scheduled once every dq CTA
// has started (D is complete by then), and it waits for the whole dq grid only before
// it exits.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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

// ---- D -------------------------------------------------------------------------------
// bwd_d_tc_kernel: one CTA per two packed row tiles (a = 2c, b = 2c + 1) of a group, so
// every K/V tile taken from L2 serves 256 rows.  Q_a, Q_b, dY_a, dY_b stay in shared
// memory; K and V tiles stream through a ring of three tile buffers (item n: the K tile
// of tile n / 2 for even n, its V tile for odd n).  TMEM: S_a 0, dP_a 128, S_b 256,
// dP_b 384; the products of one row tile run while the lanes of the other read theirs.
// Lane half h owns row tile h, one row per thread: D_i = sum_j p_ij dP_ij over all slots.
constexpr int kRing = 3;
constexpr uint32_t DQ_OFF = 0;                            // Q_a, Q_b
constexpr uint32_t DDY_OFF = 2 * kTile;                   // dY_a, dY_b
constexpr uint32_t DRING_OFF = 4 * kTile;                 // [kRing] K / V tiles
constexpr uint32_t DREL_OFF = DRING_OFF + kRing * kTile;  // float [2 stages][BT]
constexpr uint32_t DRMAX_OFF = DREL_OFF + 2 * BT * 4;     // float [2 stages][4]: max per 32 slots
constexpr uint32_t DBAR_OFF = DRMAX_OFF + 2 * 4 * 4;
enum {
  DB_Q = 0, DB_FULL0, DB_EMPTY0 = DB_FULL0 + kRing, DB_RF0 = DB_EMPTY0 + kRing,
  DB_RE0 = DB_RF0 + 2, DB_SF0 = DB_RE0 + 2, DB_SR0 = DB_SF0 + 2, DB_DONE = DB_SR0 + 2, DB_END
};
constexpr uint32_t DTMEM_OFF = DBAR_OFF + DB_END * 8;
constexpr uint32_t kSmemD = DTMEM_OFF + 16;
static_assert(kSmemD + 1024 <= 232448, "D shared memory budget");

// Positions of K tile kt relative to the chunk, and their maximum per 32 slots (one warp).
__device__ __forceinline__ void tile_rel(float *rel, float *rmax, const int32_t *tpg, int kt,
                                         int N_C, int P, int lane) {
  for (int c = 0; c < BT / 32; ++c) {
    const float v = rel_of(tpg, kt * BT + 32 * c + lane, N_C, P);  // integer-valued
    rel[32 * c + lane] = v;
    const int m = __reduce_max_sync(0xffffffffu, (int)v);
    if (lane == 0) rmax[c] = (float)m;
  }
}

__global__ void __launch_bounds__(kThr, 1)
    bwd_d_tc_kernel(const __grid_constant__ CUtensorMap q_map,
                    const __grid_constant__ CUtensorMap dy_map,
                    const __grid_constant__ CUtensorMap k_map,
                    const __grid_constant__ CUtensorMap v_map, const BwdTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  float *rel_s = reinterpret_cast<float *>(smem + DREL_OFF);
  float *rmax_s = reinterpret_cast<float *>(smem + DRMAX_OFF);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + DBAR_OFF);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + DTMEM_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rt = p.q_g * p.tiles, n_pairs = (n_rt + 1) / 2;
  const int bg = blockIdx.x / n_pairs, pr = blockIdx.x % n_pairs;
  const int b = bg / p.Hk, g = bg % p.Hk;
  const bool has_b = 2 * pr + 1 < n_rt;
  const int n_kt = p.n_kt;
  const uint64_t lim = p.timeout_ns;
  auto row_tile = [&](int h, int &bhq, int &i0) {
    const int rt = 2 * pr + h;
    bhq = b * p.Hq + g * p.q_g + rt / p.tiles;
    i0 = (rt % p.tiles) * BT;
  };
  if (threadIdx.x == 0) {
    mbar_init(&bar[DB_Q], 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&bar[DB_FULL0 + i], 1);
      mbar_init(&bar[DB_EMPTY0 + i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[DB_RF0 + s], 1);
      mbar_init(&bar[DB_RE0 + s], has_b ? kLaneWarps : kLaneWarps / 2);  // the active lane warps
      mbar_init(&bar[DB_SF0 + s], 1);
      mbar_init(&bar[DB_SR0 + s], kLaneWarps / 2);
    }
    mbar_init(&bar[DB_DONE], 1);
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
    // --------------------------- loads: Q, dY of both row tiles once; K, V, positions per tile
    const int32_t *tpg = p.token_pos + (size_t)bg * p.N_C;
    if (lane == 0) {
      mbar_expect_tx(&bar[DB_Q], (has_b ? 4 : 2) * kTile);
      for (int h = 0; h < (has_b ? 2 : 1); ++h) {
        int bhq, i0;
        row_tile(h, bhq, i0);
        tma_load_3d(smem + DQ_OFF + h * kTile, &q_map, &bar[DB_Q], 0, i0, bhq);
        tma_load_3d(smem + DQ_OFF + h * kTile + kHalf, &q_map, &bar[DB_Q], 64, i0, bhq);
        tma_load_3d(smem + DDY_OFF + h * kTile, &dy_map, &bar[DB_Q], 0, i0, bhq);
        tma_load_3d(smem + DDY_OFF + h * kTile + kHalf, &dy_map, &bar[DB_Q], 64, i0, bhq);
      }
      mbar_arrive(&bar[DB_Q]);
    }
    int n = 0;  // ring items issued
    for (int it = 0; it < n_kt && !aborted; ++it) {
      const int s = it & 1;
      if (it >= 2 && !wwait(&bar[DB_RE0 + s], ((it - 2) >> 1) & 1, lim)) { fail(p, aborted); break; }
      tile_rel(rel_s + s * BT, rmax_s + s * 4, tpg, it, p.N_C, p.P, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[DB_RF0 + s]);
      for (int u = 0; u < 2; ++u, ++n) {
        const int slot = n % kRing;
        if (n >= kRing && !wwait(&bar[DB_EMPTY0 + slot], ((n / kRing) - 1) & 1, lim)) {
          fail(p, aborted);
          break;
        }
        if (lane == 0) {
          const CUtensorMap *m = u == 0 ? &k_map : &v_map;
          mbar_expect_tx(&bar[DB_FULL0 + slot], kTile);
          tma_load_3d(smem + DRING_OFF + slot * kTile, m, &bar[DB_FULL0 + slot], 0, it * BT, bg);
          tma_load_3d(smem + DRING_OFF + slot * kTile + kHalf, m, &bar[DB_FULL0 + slot], 64, it * BT, bg);
          mbar_arrive(&bar[DB_FULL0 + slot]);
        }
      }
    }
    if (lane == 0) {  // the last loads land before exit
      mbar_wait(&bar[DB_Q], 0, 4000000000ull);
      for (int j = n - 1; j >= 0 && j >= n - kRing; --j)
        mbar_wait(&bar[DB_FULL0 + j % kRing], (j / kRing) & 1, 4000000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      if (!mbar_wait(&bar[DB_Q], 0, lim)) fail(p, aborted);
      for (int it = 0; it < n_kt && !aborted; ++it) {
        const int nk = 2 * it, nv = 2 * it + 1;
        const uint32_t k_addr = sbase + DRING_OFF + (nk % kRing) * kTile;
        const uint32_t v_addr = sbase + DRING_OFF + (nv % kRing) * kTile;
        for (int h = 0; h < (has_b ? 2 : 1); ++h) {
          // this row tile's S, dP of the previous K/V tile are read
          bool ok = it == 0 || mbar_wait(&bar[DB_SR0 + h], (it - 1) & 1, lim);
          if (ok && h == 0) ok = mbar_wait(&bar[DB_FULL0 + nk % kRing], (nk / kRing) & 1, lim);
          if (!ok) { fail(p, aborted); break; }
          tc_fence_after();
          const uint32_t q_addr = sbase + DQ_OFF + h * kTile, dy_addr = sbase + DDY_OFF + h * kTile;
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks)
            mma_bf16_ss(tmem + 256 * h, kdesc(q_addr, ks), kdesc(k_addr, ks), IDESC_KK, ks > 0);
          if (h == 0 && !mbar_wait(&bar[DB_FULL0 + nv % kRing], (nv / kRing) & 1, lim)) {
            fail(p, aborted);
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks)
            mma_bf16_ss(tmem + 256 * h + 128, kdesc(dy_addr, ks), kdesc(v_addr, ks), IDESC_KK, ks > 0);
          mma_commit(&bar[DB_SF0 + h]);
        }
        if (aborted) break;
        mma_commit(&bar[DB_EMPTY0 + nk % kRing]);  // K and V of this tile no longer read
        mma_commit(&bar[DB_EMPTY0 + nv % kRing]);
      }
      mma_commit(&bar[DB_DONE]);
      mbar_wait(&bar[DB_DONE], 0, 4000000000ull);  // drain before TMEM is freed
    }
    __syncwarp();
  } else {
    // ------------------------------------------ one row per TMEM lane; half h = row tile h
    const int half = (warp - 2) >> 2, quarter = warp & 3;
    const int r = 32 * quarter + lane;
    const uint32_t lb = (uint32_t)(32 * quarter) << 16;
    if (half == 0 || has_b) {
      int bhq, i0;
      row_tile(half, bhq, i0);
      const bool row_ok = i0 + r < p.S;
      float lse2 = row_ok ? p.lse[(size_t)bhq * p.S + i0 + r] * 1.4426950408889634f : INFINITY;
      if (!(lse2 > -INFINITY && lse2 < INFINITY)) lse2 = INFINITY;  // sees nothing / past the chunk: p = 0
      const float ri = (float)(i0 + r), rowmin = (float)(i0 + 32 * quarter);
      const float2 c22 = make_float2(p.c2, p.c2), nl22 = make_float2(-lse2, -lse2);
      float2 Dacc2 = make_float2(0.f, 0.f);
      for (int it = 0; it < n_kt && !aborted; ++it) {
        const int s = it & 1;
        if (!wwait(&bar[DB_RF0 + s], (it >> 1) & 1, lim)) { fail(p, aborted); break; }
        if (!wwait(&bar[DB_SF0 + half], it & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        const float *rel = rel_s + s * BT;
        const uint32_t cb = 256u * half;
#pragma unroll 1
        for (int c = 0; c < BT / 32; ++c) {
          uint32_t sv[32], dp[32];
          tmem_ld32(tmem + lb + cb + 32 * c, sv);
          tmem_ld32(tmem + lb + cb + 128 + 32 * c, dp);
          tmem_wait_ld();
          // a 32-slot chunk whose latest position is at or before the warp's first row is
          // seen by every row of the warp: no mask
          if (rmax_s[s * 4 + c] <= rowmin) {
#pragma unroll
            for (int e = 0; e < 32; e += 2)
              Dacc2 = fma2(ex2_2(fma2(u2f2(sv[e], sv[e + 1]), c22, nl22)), u2f2(dp[e], dp[e + 1]), Dacc2);
          } else {
            const float *rq = rel + 32 * c;
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float2 pr2 = ex2_2(fma2(u2f2(sv[e], sv[e + 1]), c22, nl22));
              pr2.x = rq[e] <= ri ? pr2.x : 0.f;
              pr2.y = rq[e + 1] <= ri ? pr2.y : 0.f;
              Dacc2 = fma2(pr2, u2f2(dp[e], dp[e + 1]), Dacc2);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar[DB_SR0 + half]);
          mbar_arrive(&bar[DB_RE0 + s]);  // slot positions no longer read
        }
      }
      if (!aborted && row_ok) p.D[(size_t)bhq * p.S + i0 + r] = Dacc2.x + Dacc2.y;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- dq --------------------------------------------------------------------------------
// bwd_dq_tc_kernel: one CTA per 128 packed rows of a group (row-stationary), D read from
// the D kernel's output.  Per K/V tile: S (columns 0 or 384 by the tile's parity) and dP
// (128); dS written back over S by 32-slot chunks (hi term, then lo term); dQ (256) +=
// dS K with dS read from TMEM, each chunk's k-steps issued once the chunk is written.
// S of the next tile is issued after the first chunk's products, dP of the next tile
// once the lanes have read all of dP, so the lanes wait only for dP.
constexpr uint32_t Q_OFF = 0, DY_OFF = kTile, K_OFF = 2 * kTile, V_OFF = 4 * kTile;
constexpr uint32_t REL_OFF = 6 * kTile;                    // float [2 stages][BT]
constexpr uint32_t RMAX_OFF = REL_OFF + 2 * BT * 4;        // float [2 stages][4]: max per 32 slots
constexpr uint32_t QBAR_OFF = RMAX_OFF + 2 * 4 * 4;
enum { QB_Q = 0, QB_KF0, QB_KE0 = QB_KF0 + 2, QB_SF0 = QB_KE0 + 2, QB_PF0 = QB_SF0 + 2, QB_DONE = QB_PF0 + 2, QB_END };
constexpr uint32_t QTMEM_OFF = QBAR_OFF + QB_END * 8;
constexpr uint32_t kSmemDq = QTMEM_OFF + 16;
static_assert(kSmemDq + 1024 <= 232448, "dq shared memory budget");

// TMEM column of the hi term of k-step kk (16 slots or rows) of a tile whose dS (or
// P) was written back by 32-wide chunks: hi of chunk c in columns 32c .. 32c + 15,
// lo 16 columns further.
__device__ __forceinline__ uint32_t a_col(int kk) { return 32u * (kk >> 1) + 8u * (kk & 1); }

__global__ void __launch_bounds__(kThr, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap q_map,
                     const __grid_constant__ CUtensorMap dy_map,
                     const __grid_constant__ CUtensorMap k_map,
                     const __grid_constant__ CUtensorMap v_map, const BwdTcParams p) {
  // D is complete (the D kernel ran before this grid): the dk/dv kernel may start as soon
  // as SMs free up
  if (threadIdx.x == 0) pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled tiles need a 1024-byte aligned base
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  float *rel_s = reinterpret_cast<float *>(smem + REL_OFF);
  float *rmax_s = reinterpret_cast<float *>(smem + RMAX_OFF);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + QBAR_OFF);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + QTMEM_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rt = p.q_g * p.tiles;
  const int bg = blockIdx.x / n_rt, rt = blockIdx.x % n_rt;
  const int b = bg / p.Hk, g = bg % p.Hk;
  const int hl = rt / p.tiles, t = rt % p.tiles;
  const int bhq = b * p.Hq + g * p.q_g + hl, i0 = t * BT;
  const int n_kt = p.n_kt;
  const uint64_t lim = p.timeout_ns;
  if (threadIdx.x == 0) {
    mbar_init(&bar[QB_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[QB_KF0 + s], 1);
      mbar_init(&bar[QB_KE0 + s], 1 + kLaneWarps);  // MMA commit + the lane warps (positions)
      mbar_init(&bar[QB_SF0 + s], 1);
      mbar_init(&bar[QB_PF0 + s], kLaneWarps);
    }
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
    for (; it < n_kt && !aborted; ++it) {
      const int s = it & 1, use = it >> 1;
      if (use > 0 && !wwait(&bar[QB_KE0 + s], (use - 1) & 1, lim)) { fail(p, aborted); break; }
      tile_rel(rel_s + s * BT, rmax_s + s * 4, tpg, it, p.N_C, p.P, lane);
      __syncwarp();
      if (lane == 0) {
        mbar_expect_tx(&bar[QB_KF0 + s], 2 * kTile);
        tma_load_3d(smem + K_OFF + s * kTile, &k_map, &bar[QB_KF0 + s], 0, it * BT, bg);
        tma_load_3d(smem + K_OFF + s * kTile + kHalf, &k_map, &bar[QB_KF0 + s], 64, it * BT, bg);
        tma_load_3d(smem + V_OFF + s * kTile, &v_map, &bar[QB_KF0 + s], 0, it * BT, bg);
        tma_load_3d(smem + V_OFF + s * kTile + kHalf, &v_map, &bar[QB_KF0 + s], 64, it * BT, bg);
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
      auto kv_addr = [&](int st, uint32_t off) { return sbase + off + st * kTile; };
      auto issue_s = [&](int st, uint32_t col) {  // S = Q K^T
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks)
          mma_bf16_ss(tmem + col, kdesc(q_addr, ks), kdesc(kv_addr(st, K_OFF), ks), IDESC_KK, ks > 0);
      };
      auto issue_dp = [&](int st, uint32_t col) {  // dP = dY V^T
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks)
          mma_bf16_ss(tmem + col, kdesc(dy_addr, ks), kdesc(kv_addr(st, V_OFF), ks), IDESC_KK, ks > 0);
      };
      // dQ += dS K over the k-steps of chunk qq of both lane halves (slots 32 qq .. and
      // 64 + 32 qq ..), dS read from TMEM at column xs (two bf16 per column)
      auto dq_products = [&](int st, uint32_t xs, int qq, bool first) {
        const uint32_t k_addr = kv_addr(st, K_OFF);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int kk = 2 * qq + (u & 1) + 4 * (u >> 1);
          mma_bf16_ts(tmem + 256, tmem + xs + a_col(kk), mdesc(k_addr, kk), IDESC_TM,
                      (first && u == 0) ? 0u : 1u);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int kk = 2 * qq + (u & 1) + 4 * (u >> 1);
          mma_bf16_ts(tmem + 256, tmem + xs + a_col(kk) + 16, mdesc(k_addr, kk), IDESC_TM, 1u);
        }
      };
      bool ok = mbar_wait(&bar[QB_Q], 0, lim) && mbar_wait(&bar[QB_KF0], 0, lim);
      if (!ok) {
        fail(p, aborted);
      } else {
        tc_fence_after();
        issue_s(0, 0);
        issue_dp(0, 128);
        mma_commit(&bar[QB_SF0]);
      }
      for (int m = 0; m < n_kt && !aborted; ++m) {
        const int s = m & 1;
        const uint32_t xs = (m & 1) ? 384u : 0u;
        const bool more = m + 1 < n_kt;
        if (!mbar_wait(&bar[QB_PF0], m & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        dq_products(s, xs, 0, m == 0);
        if (more) {
          if (!mbar_wait(&bar[QB_KF0 + (s ^ 1)], ((m + 1) >> 1) & 1, lim)) { fail(p, aborted); break; }
          tc_fence_after();
          issue_s(s ^ 1, xs ^ 384u);
        }
        if (!mbar_wait(&bar[QB_PF0 + 1], m & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        if (more) {
          issue_dp(s ^ 1, 128);
          mma_commit(&bar[QB_SF0 + (s ^ 1)]);
        }
        dq_products(s, xs, 1, false);
        mma_commit(&bar[QB_KE0 + s]);  // K, V of this stage no longer read
      }
      mma_commit(&bar[QB_DONE]);
      mbar_wait(&bar[QB_DONE], 0, 4000000000ull);  // drain before TMEM is freed
    }
    __syncwarp();
  } else {
    // ----------------- one row per TMEM lane; two warps per lane quarter split the slots
    const int half = (warp - 2) >> 2, quarter = warp & 3;
    const int r = 32 * quarter + lane;
    const uint32_t lb = (uint32_t)(32 * quarter) << 16;
    const bool row_ok = i0 + r < p.S;
    float lse2 = row_ok ? p.lse[(size_t)bhq * p.S + i0 + r] * 1.4426950408889634f : INFINITY;
    if (!(lse2 > -INFINITY && lse2 < INFINITY)) lse2 = INFINITY;  // sees nothing / past the chunk: p = 0
    const float D = row_ok ? __ldcg(p.D + (size_t)bhq * p.S + i0 + r) : 0.f;
    const float ri = (float)(i0 + r), rowmin = (float)(i0 + 32 * quarter);
    const float2 c22 = make_float2(p.c2, p.c2), nl22 = make_float2(-lse2, -lse2);
    const float2 nD2 = make_float2(-D, -D);
    for (int it = 0; it < n_kt && !aborted; ++it) {
      const int s = it & 1, use = it >> 1;
      if (!wwait(&bar[QB_SF0 + s], use & 1, lim)) { fail(p, aborted); break; }
      if (!wwait(&bar[QB_KF0 + s], use & 1, lim)) { fail(p, aborted); break; }
      tc_fence_after();
      const float *rel = rel_s + s * BT + 64 * half;  // this half's 64 slots
      // dS by 32-slot chunks, written back over the chunk's S columns (S at column 0 or
      // 384 by the tile's parity): hi term in the first 16, lo term in the next 16
      const uint32_t xs = (it & 1) ? 384u : 0u;
#pragma unroll 1
      for (int qq = 0; qq < 2; ++qq) {
        const uint32_t c0 = 64u * half + 32u * qq;
        uint32_t sv[32], dp[32], hi[16], lo[16];
        tmem_ld32(tmem + lb + xs + c0, sv);
        tmem_ld32(tmem + lb + 128 + c0, dp);
        tmem_wait_ld();
        if (rmax_s[s * 4 + 2 * half + qq] <= rowmin) {  // every row of the warp sees the chunk
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 pr = ex2_2(fma2(u2f2(sv[e], sv[e + 1]), c22, nl22));
            split2(mul2(pr, add2(u2f2(dp[e], dp[e + 1]), nD2)), hi[e >> 1], lo[e >> 1]);
          }
        } else {
          const float *rq = rel + 32 * qq;
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float2 pr = ex2_2(fma2(u2f2(sv[e], sv[e + 1]), c22, nl22));
            pr.x = rq[e] <= ri ? pr.x : 0.f;
            pr.y = rq[e + 1] <= ri ? pr.y : 0.f;
            split2(mul2(pr, add2(u2f2(dp[e], dp[e + 1]), nD2)), hi[e >> 1], lo[e >> 1]);
          }
        }
        tmem_st16(tmem + lb + xs + c0, hi);
        tmem_st16(tmem + lb + xs + c0 + 16, lo);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar[QB_PF0 + qq]);
          if (qq == 1) mbar_arrive(&bar[QB_KE0 + s]);  // slot positions no longer read
        }
      }
    }
    if (!aborted && wwait(&bar[QB_DONE], 0, lim)) {
      tc_fence_after();
      float *dst = p.dq + ((size_t)bhq * p.S + i0 + r) * HD + 64 * half;
#pragma unroll 1
      for (int cq = 0; cq < 2; ++cq) {
        uint32_t o[32];
        tmem_ld32(tmem + lb + 256 + 64 * half + 32 * cq, o);
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
constexpr uint32_t ROWS_OFF = 6 * kTile;                     // float [2 stages][2][BT]: -lse2, -D
constexpr uint32_t KBAR_OFF = ROWS_OFF + 2 * 2 * BT * 4;
enum { KB_KV = 0, KB_QF0, KB_QE0 = KB_QF0 + 2, KB_SF = KB_QE0 + 2, KB_PF0, KB_DONE = KB_PF0 + 2, KB_END };
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
      mbar_init(&bar[KB_QE0 + s], 1 + kLaneWarps);  // MMA commit + the lane warps (lse2, D)
      mbar_init(&bar[KB_PF0 + s], kLaneWarps);
    }
    mbar_init(&bar[KB_SF], 1);
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
        rows_s[(s * 2 + 0) * BT + r] = -l2;
        rows_s[(s * 2 + 1) * BT + r] = ok ? -__ldcg(p.D + (size_t)bhq * p.S + i0 + r) : 0.f;
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
        // dV += P^T dY, dK += dS^T Q (A from TMEM: P^T terms in columns 0 .., dS^T terms
        // in 128 ..; B: the row tiles as MN-major operands), the k-steps of each lane
        // half's first 32 rows once PF0 completes, the rest after PF1
        for (int qq = 0; qq < 2 && !aborted; ++qq) {
          if (!mbar_wait(&bar[KB_PF0 + qq], it & 1, lim)) { fail(p, aborted); break; }
          tc_fence_after();
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int kk = 2 * qq + (u & 1) + 4 * (u >> 1);
            mma_bf16_ts(tmem + 256, tmem + a_col(kk), mdesc(dy_addr, kk), IDESC_TM,
                        (it > 0 || qq > 0 || u > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int kk = 2 * qq + (u & 1) + 4 * (u >> 1);
            mma_bf16_ts(tmem + 256, tmem + a_col(kk) + 16, mdesc(dy_addr, kk), IDESC_TM, 1u);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int kk = 2 * qq + (u & 1) + 4 * (u >> 1);
            mma_bf16_ts(tmem + 384, tmem + 128 + a_col(kk), mdesc(q_addr, kk), IDESC_TM,
                        (it > 0 || qq > 0 || u > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int kk = 2 * qq + (u & 1) + 4 * (u >> 1);
            mma_bf16_ts(tmem + 384, tmem + 128 + a_col(kk) + 16, mdesc(q_addr, kk), IDESC_TM, 1u);
          }
        }
        if (aborted) break;
        mma_commit(&bar[KB_QE0 + s]);  // Q, dY of this stage no longer read
      }
      mma_commit(&bar[KB_DONE]);
      mbar_wait(&bar[KB_DONE], 0, 4000000000ull);
    }
    __syncwarp();
  } else {
    // ---------------- one slot per TMEM lane; two warps per lane quarter split the rows
    const int half = (warp - 2) >> 2, quarter = warp & 3;
    const int jl = 32 * quarter + lane;
    const int j = kt * BT + jl;
    const uint32_t lb = (uint32_t)(32 * quarter) << 16;
    const float rel = rel_of(p.token_pos + (size_t)bg * p.N_C, j, p.N_C, p.P);
    const float2 c22 = make_float2(p.c2, p.c2);
    for (int it = 0; it < n_rt && !aborted; ++it) {
      const int s = it & 1, use = it >> 1;
      const int t = it % p.tiles, i0 = t * BT;
      if (!wwait(&bar[KB_SF], it & 1, lim)) { fail(p, aborted); break; }
      if (!wwait(&bar[KB_QF0 + s], use & 1, lim)) { fail(p, aborted); break; }
      tc_fence_after();
      // row r of the tile sees this slot iff i0 + r >= rel; rows past the chunk have
      // -lse2 = -inf
      const float rmin = rel - (float)i0;
      const float *nl2 = rows_s + (s * 2 + 0) * BT, *nD = rows_s + (s * 2 + 1) * BT;
      // by chunks of 32 rows (S^T columns r0 .. r0 + 31), written back over the
      // chunk's own columns: P^T hi, lo in r0 .., r0 + 16 ..; dS^T hi, lo 128 further
#pragma unroll 1
      for (int qq = 0; qq < 2; ++qq) {
        const int r0 = 64 * half + 32 * qq;
        uint32_t sv[32], dp[32], phi[16], plo[16], dhi[16], dlo[16];
        tmem_ld32(tmem + lb + r0, sv);
        tmem_ld32(tmem + lb + 128 + r0, dp);
        tmem_wait_ld();
        if (__all_sync(0xffffffffu, rmin <= (float)r0)) {  // every row sees every slot of the warp
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 pr =
                ex2_2(fma2(u2f2(sv[e], sv[e + 1]), c22, *reinterpret_cast<const float2 *>(nl2 + r0 + e)));
            split2(pr, phi[e >> 1], plo[e >> 1]);
            split2(mul2(pr, add2(u2f2(dp[e], dp[e + 1]), *reinterpret_cast<const float2 *>(nD + r0 + e))),
                   dhi[e >> 1], dlo[e >> 1]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int r = r0 + e;
            float2 pr = ex2_2(fma2(u2f2(sv[e], sv[e + 1]), c22, *reinterpret_cast<const float2 *>(nl2 + r)));
            pr.x = (float)r >= rmin ? pr.x : 0.f;
            pr.y = (float)(r + 1) >= rmin ? pr.y : 0.f;
            split2(pr, phi[e >> 1], plo[e >> 1]);
            split2(mul2(pr, add2(u2f2(dp[e], dp[e + 1]), *reinterpret_cast<const float2 *>(nD + r))),
                   dhi[e >> 1], dlo[e >> 1]);
          }
        }
        tmem_st16(tmem + lb + r0, phi);
        tmem_st16(tmem + lb + r0 + 16, plo);
        tmem_st16(tmem + lb + 128 + r0, dhi);
        tmem_st16(tmem + lb + 128 + r0 + 16, dlo);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar[KB_PF0 + qq]);
          if (qq == 1) mbar_arrive(&bar[KB_QE0 + s]);  // -lse2, -D of this stage no longer read
        }
      }
    }
    if (!aborted && wwait(&bar[KB_DONE], 0, lim)) {
      tc_fence_after();
      // half 0 writes dV, half 1 dK
      const bool ok = j < p.N_C;
      float *dst = (half == 0 ? p.dv : p.dk) + ((size_t)bg * p.N_C + j) * HD;
      const float f = half == 0 ? 1.f : p.rsd;
#pragma unroll 1
      for (int cq = 0; cq < 4; ++cq) {
        uint32_t o[32];
        tmem_ld32(tmem + lb + 256 + 128 * half + 32 * cq, o);
        tmem_wait_ld();
        if (ok) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4 *>(dst + 32 * cq)[e] =
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
  if (threadIdx.x == 0) pdl_wait();  // complete only after the dq grid (stream order)
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
  static thread_local bool done_d = false, done_q = false, done_kv = false;
  int dev = 0;
  cudaGetDevice(&dev);
  if (ready_dev != dev) {
    done_d = done_q = done_kv = false;
    ready_dev = dev;
  }
  rc = opt_in(bwd_d_tc_kernel, kSmemD + 1024, done_d);
  if (rc) return rc;
  rc = opt_in(bwd_dq_tc_kernel, kSmemDq + 1024, done_q);
  if (rc) return rc;
  rc = opt_in(bwd_dkdv_tc_kernel, kSmemKv + 1024, done_kv);
  if (rc) return rc;
  const CUtensorMap &kmap = *reinterpret_cast<const CUtensorMap *>(c->tc.k_map);
  const CUtensorMap &vmap = *reinterpret_cast<const CUtensorMap *>(c->tc.v_map);
  const long long groups = (long long)d.batch * d.n_kv_heads;
  const long long n_rt = (long long)p.q_g * p.tiles;
  const long long g_d = groups * ((n_rt + 1) / 2), g_dq = groups * n_rt, g_kv = groups * p.n_kt;
  if (g_dq > INT32_MAX || g_kv > INT32_MAX)
    return set_error(H2OKV_ERR_UNSUPPORTED, "backward grid too large");
  bwd_d_tc_kernel<<<(unsigned)g_d, kThr, kSmemD + 1024, st>>>(qmap, dymap, kmap, vmap, p);
  rc = check_launch("bwd_d_tc_kernel");
  if (rc) return rc;
  bwd_dq_tc_kernel<<<(unsigned)g_dq, kThr, kSmemDq + 1024, st>>>(qmap, dymap, kmap, vmap, p);
  rc = check_launch("bwd_dq_tc_kernel");
  if (rc) return rc;
  // dk/dv as a programmatic dependent of dq: its CTAs fill the SMs that dq's last wave
  // leaves idle (D is complete before dq starts)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)g_kv);
  cfg.blockDim = dim3(kThr);
  cfg.dynamicSmemBytes = kSmemKv + 1024;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, bwd_dkdv_tc_kernel, qmap, dymap, kmap, vmap, p);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "bwd_dkdv_tc_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("bwd_dkdv_tc_kernel");
}

}  // namespace h2okv
