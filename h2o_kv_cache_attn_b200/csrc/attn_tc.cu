// Tensor-core path of chunked cache attention with summed weights for d = 128
// and a bf16, int8 or int4 cache ("Learning how to Forget", §A.1 token-position
// mask, §A.7 SDPA plus the attention weights summed over the query axis, returned
// per KV slot and summed over the q_g query heads of each GQA group; §4 / Table
// 1 8- and 4-bit caches).
//
// A CTA owns two 128-row query tiles (a, b) of one KV group (two row tiles of
// one head, or the same rows of two heads); rows past S are zero-filled by TMA
// and never written.  Each 128-slot K/V tile is read once for both query tiles.
// The warp roles: warp 0 loads Q and K tiles (cp.async.bulk.tensor, no multicast)
// and the slots' token positions, warp 2 loads V tiles, warp 1 allocates TMEM and
// issues every MMA from one thread, warps 4-7 (tile a) and 8-11 (tile b) own TMEM
// lanes 32(w%4)..32(w%4)+31 for the softmax, the column sums and the epilogue.
//
// bf16 caches run two passes:
//   attn_fwd_kernel   S = Q K^T (tcgen05.mma, M=128 rows, N=128 slots, fp32 in TMEM);
//                     online softmax per row against a lazily moved reference
//                     maximum; P written over S in TMEM as bf16 pairs; O += P V
//                     with P read from TMEM (A) and V from shared memory (B).
//                     Writes y and -lse2 per row (combine_fwd_kernel merges the
//                     pieces of pairs split over CTAs).
//   scoresum_kernel   S^T = K Q^T (M=128 slots, N=128 rows): one thread per SLOT
//                     forms p = exp2(s*log2e/sqrt(d) - lse2_i) with the FINAL row
//                     LSE and sums them in registers (no atomics, deterministic),
//                     over equal shares of the (pair, K tile) units on every SM.
// attn_tc_kernel runs both phases in one CTA (phase A: online max / sum -> LSE;
// phase B: S^T with the final LSE, column sums, P in shared memory, O += P V) and
// serves the int8 / int4 caches: there warps 0, 2, 3 and 12-15 replace the TMA
// producers, stage each tile of codes by a bulk copy and dequantize it in place
// (see convert_i8 / convert_i4): key tiles become exact f16 integers and the key
// scale s_j multiplies the logits of slot j, so scores and summed weights see the
// stored keys exactly; value tiles are stored as bf16(code * scale).
// Every wait is bounded; a timeout sets the cache's device status word and the
// CTA drains its copies and MMAs before freeing TMEM.
//
// Per-(query tile, slot) sums go to a partial buffer; a small reduction kernel
// sums them in a fixed order into w [B, H_k, N_C] and wq [B, H_q, N_C].
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "h2okv_internal.cuh"
#include "tc_ptx.cuh"

namespace h2okv {
namespace {

using namespace ptx;

constexpr int BM = 128;        // query rows per tile
constexpr int BN = 128;        // slots per tile
constexpr int D = 128;         // head dim
constexpr int kThreads = 384;  // 4 control warps + 2 softmax warpgroups
constexpr int kPrefetch = 4;   // K / V tiles requested into L2 this many loads ahead
constexpr int kRelFar = 1 << 20;  // relative position of a slot no row of the chunk sees
constexpr float kMaskBias = 1073741824.f;  // 2^30: a masked logit drops by this (base-2 units)
// Register split between the warpgroups.  The launch allots 168 registers per
// thread (384 x 168 = 64512); the control warpgroup drops to 88 and the two
// softmax warpgroups rise to 208: 128 x 88 + 256 x 208 = 64512.
constexpr int kLaunchRegs = 168, kCtrlRegs = 88, kSoftRegs = 208;
static_assert(128 * kCtrlRegs + 256 * kSoftRegs == kThreads * kLaunchRegs, "register split");
// Quantized caches: 512 threads, warps 12-15 join the loaders.  Launch allotment 128
// registers (512 x 128 = 65536); the control and loader warpgroups drop to 64, the
// softmax warpgroups rise to 192: 256 x 64 + 256 x 192 = 65536.
constexpr int kThreadsQ = 512;
constexpr int kLaunchRegsQ = 128, kCtrlRegsQ = 64, kSoftRegsQ = 192;
static_assert(256 * kCtrlRegsQ + 256 * kSoftRegsQ == kThreadsQ * kLaunchRegsQ, "register split");
template <int KV>
__host__ __device__ constexpr int threads_of() { return KV == H2OKV_BF16 ? kThreads : kThreadsQ; }
template <int KV>
__host__ __device__ constexpr int launch_regs_of() {
  return KV == H2OKV_BF16 ? kLaunchRegs : kLaunchRegsQ;
}
constexpr uint32_t kTileBytes = BM * D * 2;  // 32 KiB (two 64-column swizzled halves)
constexpr uint32_t kHalfBytes = kTileBytes / 2;

// shared memory carve-up (1024-aligned base)
constexpr uint32_t OFF_QA = 0;
constexpr uint32_t OFF_QB = OFF_QA + kTileBytes;
constexpr uint32_t OFF_K0 = OFF_QB + kTileBytes;
constexpr uint32_t OFF_K1 = OFF_K0 + kTileBytes;
constexpr uint32_t OFF_V0 = OFF_K1 + kTileBytes;
constexpr uint32_t OFF_V1 = OFF_V0 + kTileBytes;
constexpr uint32_t OFF_P = OFF_V1 + kTileBytes;
constexpr uint32_t OFF_TP = OFF_P + kTileBytes;        // int32 [2 stages][BN]
constexpr uint32_t OFF_LSE = OFF_TP + 2 * BN * 4;      // float [2 tiles][BM]
constexpr uint32_t OFF_KSB = OFF_LSE + 2 * BM * 4;     // fp16 [2 stages][BN] phase B key scales
constexpr uint32_t OFF_BAR = OFF_KSB + 2 * BN * 2;     // uint64 barriers
constexpr int kStagesA = 4;  // phase A K ring: slots K0, K1, V0, V1 (V is unused in phase A)
constexpr int NBAR = 25 + 2 * kStagesA + 5;
constexpr uint32_t OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr uint32_t kSmemBytes = OFF_TMEM + 16;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// phase A stage -> slot; phase A token positions (float [kStagesA][BN]) and key
// scales (float [kStagesA][BN], quantized caches) live in the P region, unused in phase A
constexpr uint32_t OFF_REL_A = OFF_P;
constexpr uint32_t OFF_KS_A = OFF_P + kStagesA * BN * 4;
__host__ __device__ constexpr uint32_t slot_a(int a) {
  return a == 0 ? OFF_K0 : a == 1 ? OFF_K1 : a == 2 ? OFF_V0 : OFF_V1;
}
// last phase A tile that used stage a (or -1): the slot is free once that use is released
__device__ __forceinline__ int last_use_a(int a, int n_kt) {
  if (a >= n_kt) return -1;
  return a + ((n_kt - 1 - a) / kStagesA) * kStagesA;
}

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t IDESC_K_MAJOR = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t IDESC_K_MAJOR_F16 = idesc_f16_f32(128, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, true, true);

struct TcParams {
  const int32_t *token_pos;  // [B*Hk][N_C]
  const uint8_t *kq, *vq;    // quantized caches: codes [B*Hk][N_C][row bytes]
  const __half *ksc, *vsc;   // quantized caches: scales [B*Hk][N_C]
  __nv_bfloat16 *y;          // [B*Hq][S][D]
  float *lse_out;            // [B*Hq][S] or null
  float *part_w;             // [B*Hq*tiles][N_C]
  float *nlse;               // [B*Hq*tiles][BM]: -lse2 of every row (bf16 two-pass path)
  int *status;               // device status word (0 = ok)
  int Hq, Hk, q_g, N_C, S, P, tiles, n_kt, ctas_per_group;
  float scale2;  // log2(e) / sqrt(d)
  unsigned long long timeout_ns;
};

enum {
  B_Q = 0,
  B_KFULL0, B_KFULL1, B_KEMPTY0, B_KEMPTY1,  // phase B K ring (+ token positions)
  B_VFULL0, B_VFULL1, B_VEMPTY0, B_VEMPTY1,  // V ring (phase B)
  B_SFULL0, B_SFULL1, B_SFREE0, B_SFREE1,    // phase A S pair per tile parity
  B_AFREE,                                   // phase A TMEM fully read
  B_TFULLA, B_TFULLB, B_TFREEA, B_TFREEB,    // phase B S^T per query tile
  B_PFULLA, B_PFULLB, B_PFREEA, B_PFREEB,    // P buffer, handed a(kt) -> b(kt) -> a(kt+1)
  B_OFULL, B_DRAIN,                          // O complete; MMA drain before TMEM is freed
  B_VGO,                                     // every phase A MMA done: V may use slots V0 / V1
  B_AFULL0, B_AEMPTY0 = B_AFULL0 + kStagesA,  // phase A K ring (+ token positions)
  B_LOADED0 = B_AEMPTY0 + kStagesA,          // quantized caches: codes staged in K0, K1, V0, V1
  B_QREADY = B_LOADED0 + 4,                  // quantized caches: Q tiles converted to fp16
  B_END = B_QREADY + 1
};
static_assert(B_END == NBAR, "barrier count");

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

// Masking of one row of raw logits: a masked logit (slot relative position rel_e >
// row index ri) drops by mbias = 2^30 / (logit scale), i.e. by 2^30 in base-2 units;
// nm = sat(rel_e - ri) is 1 for a masked slot, 0 for a visible one.
template <int N>
__device__ __forceinline__ void row_mask(uint32_t (&x)[N], const float *rel, float ri,
                                         float mbias) {
#pragma unroll
  for (int e = 0; e < N; e += 4) {
    const float4 r4 = *reinterpret_cast<const float4 *>(rel + e);
    const float rr[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float nm = fma_sat(rr[q], 1.f, -ri);
      x[e + q] = __float_as_uint(fmaf(nm, -mbias, __uint_as_float(x[e + q])));
    }
  }
}

// Online (max, sum) update of one row over N slots (base-2 units).
template <int N>
__device__ __forceinline__ void row_update(const uint32_t (&x)[N], float c2, float &m, float &l) {
  static_assert(N % 16 == 0, "row width");
  float mx8[8];  // eight independent chains of three-input maxima
#pragma unroll
  for (int q = 0; q < 8; ++q) mx8[q] = fmaxf(__uint_as_float(x[q]), __uint_as_float(x[q + 8]));
#pragma unroll
  for (int e = 16; e < N; e += 16) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      mx8[q] = fmax3(mx8[q], __uint_as_float(x[e + q]), __uint_as_float(x[e + 8 + q]));
  }
  const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                         fmaxf(mx8[6], mx8[7]));
  const float m_new = fmaxf(m, mx * c2);
  if (m_new == -INFINITY) return;
  const float2 c2v = make_float2(c2, c2), negm = make_float2(-m_new, -m_new);
  float2 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
  for (int e = 0; e < N; e += 2) {
    const float2 a =
        fma2(make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])), c2v, negm);
    const float2 v = make_float2(ex2(a.x), ex2(a.y));
    acc[(e >> 1) & 3] = add2(acc[(e >> 1) & 3], v);
  }
  const float2 s01 = add2(acc[0], acc[1]), s23 = add2(acc[2], acc[3]);
  const float2 s4 = add2(s01, s23);
  l = l * ex2(m - m_new) + (s4.x + s4.y);
  m = m_new;
}

// Phase B for one slot (this thread) and one query tile: normalised p over the
// tile's 128 rows from S^T in TMEM, packed to bf16 pairs, column sum returned.
// nlse holds -lse2 of the tile's rows.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[BM]) {
  tmem_ld32(taddr + 0, *reinterpret_cast<uint32_t(*)[32]>(r + 0));
  tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
  tmem_ld32(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(r + 64));
  tmem_ld32(taddr + 96, *reinterpret_cast<uint32_t(*)[32]>(r + 96));
  tmem_wait_ld();
}

__device__ __forceinline__ float slot_probs(const uint32_t (&r)[BM], const float *nlse, float c2,
                                            int rmin, int rmax, bool full, uint32_t (&pk)[BM / 2]) {
  const float rminf = (float)rmin;
  const float2 c2v = make_float2(c2, c2);
  float2 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
  for (int e = 0; e < BM; e += 2) {
    const float2 nl = *reinterpret_cast<const float2 *>(nlse + e);
    float2 a = fma2(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), c2v, nl);
    if (!full) {  // rows before rmin are masked: nm = sat(rmin - row) is 1 there
      const float2 nm = make_float2(fma_sat(rminf, 1.f, -(float)e), fma_sat(rminf, 1.f, -(float)(e + 1)));
      a = fma2(nm, make_float2(-kMaskBias, -kMaskBias), a);
    }
    float2 v = make_float2(ex2(a.x), ex2(a.y));
    if (rmax < BM) {  // rows past the chunk (last row tile only)
      v.x = e < rmax ? v.x : 0.f;
      v.y = e + 1 < rmax ? v.y : 0.f;
    }
    acc[(e >> 1) & 3] = add2(acc[(e >> 1) & 3], v);
    pk[e >> 1] = pack_bf16x2(v.x, v.y);
  }
  const float2 s01 = add2(acc[0], acc[1]), s23 = add2(acc[2], acc[3]);
  const float2 s4 = add2(s01, s23);
  return s4.x + s4.y;
}

// P[row][slot] as the MN-major A operand: slot = K index (a 128-byte row of an
// 8-slot atom), rows = M index (64 per block, 16-byte chunks swizzled).
__device__ __forceinline__ void store_p(uint32_t p_slot_row, int st, const uint32_t (&pk)[BM / 2]) {
#pragma unroll
  for (int mb = 0; mb < 2; ++mb) {
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const int base = mb * 32 + cc * 4;
      const uint32_t addr = p_slot_row + mb * kHalfBytes + ((cc ^ (st & 7)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[base]),
                   "r"(pk[base + 1]), "r"(pk[base + 2]), "r"(pk[base + 3])
                   : "memory");
    }
  }
}

// ---- quantized caches: dequantizing tile loads --------------------------------------
// One loader thread copies a 128-slot tile of codes with a bulk copy into the upper
// 16 KiB of the bf16 operand buffer it becomes; the 96 loader threads (warps 0, 2, 3)
// then turn every code into bf16 in place and store the tile in the swizzled K-major
// layout the MMA reads (the bytes a TMA load of a bf16 tile would produce: row j at
// 128 j, 16-byte chunk c at c ^ (j % 8), dims 64..127 in the second 16 KiB half).
// A code c becomes a float exactly as the float whose bits are 0x4B0000uu (2^23 + u,
// u = c + 128 or c + 8 as an unsigned byte) minus 2^23 + 128 (or + 8); |c| <= 127
// is exact in bf16.  Value tiles are multiplied by their slot's scale first (exact
// in float32, one rounding to bf16).
constexpr int kLoaderWarps = 7;  // warps 0, 2, 3 and 12-15
constexpr int kConvThreads = 32 * kLoaderWarps;
constexpr uint32_t kStageOff = kHalfBytes;  // staged codes: upper half of the buffer
template <int KV>
struct QTile;
template <>
struct QTile<H2OKV_I8> {
  static constexpr int kRowBytes = D;
};
template <>
struct QTile<H2OKV_I4> {
  static constexpr int kRowBytes = D / 2;
};

__device__ __forceinline__ float offset_byte_float(uint32_t u, uint32_t k) {
  return __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7440u | k));  // bits 0x4B0000 | byte k
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// 8 int8 codes (element 4i + k in byte k of word i) -> 4 bf16 pairs in element order
__device__ __forceinline__ void cvt_i8x8(uint32_t w0, uint32_t w1, float2 s2, bool fold,
                                         uint32_t (&o)[4]) {
  const float2 off = make_float2(-8388736.f, -8388736.f);  // -(2^23 + 128)
  const uint32_t ws[2] = {w0 ^ 0x80808080u, w1 ^ 0x80808080u};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float2 a = add2(make_float2(offset_byte_float(ws[i], 0), offset_byte_float(ws[i], 1)), off);
    float2 b = add2(make_float2(offset_byte_float(ws[i], 2), offset_byte_float(ws[i], 3)), off);
    if (fold) {
      a = mul2(a, s2);
      b = mul2(b, s2);
    }
    o[2 * i] = pack_bf16x2(a.x, a.y);
    o[2 * i + 1] = pack_bf16x2(b.x, b.y);
  }
}

// 8 int4 codes (element 2k in the low nibble, 2k + 1 in the high nibble of byte k)
// -> 4 bf16 pairs in element order
__device__ __forceinline__ void cvt_i4x8(uint32_t w, float2 s2, bool fold, uint32_t (&o)[4]) {
  const float2 off = make_float2(-8388616.f, -8388616.f);  // -(2^23 + 8)
  const uint32_t u = w ^ 0x88888888u;
  const uint32_t lo = u & 0x0F0F0F0Fu, hi = (u >> 4) & 0x0F0F0F0Fu;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float2 a = add2(make_float2(offset_byte_float(lo, k), offset_byte_float(hi, k)), off);
    if (fold) a = mul2(a, s2);
    o[k] = pack_bf16x2(a.x, a.y);
  }
}

// Keys of quantized caches enter the logit MMAs as f16 (exact for |code| <= 127).
// 8 int8 codes -> 4 f16 pairs in element order: the f16 with bits 0x64uu is 1024 + u.
__device__ __forceinline__ void cvt_i8_f16x8(uint32_t w0, uint32_t w1, uint32_t (&o)[4]) {
  const uint32_t u0 = w0 ^ 0x80808080u, u1 = w1 ^ 0x80808080u;
  const uint32_t t[4] = {__byte_perm(u0, 0x64646464u, 0x4140u), __byte_perm(u0, 0x64646464u, 0x4342u),
                         __byte_perm(u1, 0x64646464u, 0x4140u), __byte_perm(u1, 0x64646464u, 0x4342u)};
  const __half2 off = __float2half2_rn(1152.f);  // 1024 + 128
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2 h = __hsub2(*reinterpret_cast<const __half2 *>(&t[k]), off);
    o[k] = *reinterpret_cast<const uint32_t *>(&h);
  }
}
// 8 int4 codes (element n in nibble n) -> 4 f16 pairs in the order (0, 4) (1, 5) (2, 6)
// (3, 7); the query tile's chunks are reordered the same way, so the dot products are
// unchanged.
__device__ __forceinline__ void cvt_i4_f16x8(uint32_t w, uint32_t (&o)[4]) {
  const uint32_t u = w ^ 0x88888888u;
  const __half2 off = __float2half2_rn(1032.f);  // 1024 + 8
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t t = ((u >> (4 * k)) & 0x000F000Fu) | 0x64006400u;
    const __half2 h = __hsub2(*reinterpret_cast<const __half2 *>(&t), off);
    o[k] = *reinterpret_cast<const uint32_t *>(&h);
  }
}

// Exponent e of the power of two a query tile is divided by before it becomes f16:
// its largest |q| (float bits maxbits) then lies in [2^14, 2^15).
__device__ __forceinline__ int q_exponent(uint32_t maxbits) {
  if (maxbits == 0u) return 0;
  const int lg = (int)((maxbits >> 23) & 0xFFu) - 127;
  return min(max(lg - 14, -100), 100);
}
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// int8 in place (keys to exact f16, values to bf16(code * scale)): the staged code
// row j (128 bytes at kStageOff + 128 j) occupies the
// bytes of bf16 row j of the upper half, so each warp owns whole rows (4 per pass: 8
// lanes of 16 codes per row) and reads a pass's rows before any lane rewrites them;
// no other warp's rows are touched.  w3 is this warp's index among the loader warps;
// sv[i] is the value scale of this lane's row in pass i (values only).  Rows at or
// past nv (outside the cache) are written as zeros.
constexpr int kI8Passes = (32 + kLoaderWarps - 1) / kLoaderWarps;  // 32 groups of 4 rows
__device__ __forceinline__ void convert_i8(uint32_t buf, int nv, const float (&sv)[kI8Passes + 1],
                                           bool fold, int w3, int lane) {
  const int q = lane & 7;
  constexpr int kU = 4;  // passes in flight
#pragma unroll
  for (int it = 0; it < kI8Passes; it += kU) {
    uint4 w[kU];
    int row[kU];
    bool act[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int g = w3 + kLoaderWarps * (it + u);
      act[u] = it + u < kI8Passes && g < 32;
      row[u] = 4 * g + (lane >> 3);
      w[u] = make_uint4(0u, 0u, 0u, 0u);
      if (act[u] && row[u] < nv) w[u] = ld_shared_v4(buf + kStageOff + row[u] * 128 + q * 16);
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (!act[u]) continue;
      const float s1 = it + u < kI8Passes ? sv[it + u] : 0.f;
      const float2 s2 = make_float2(s1, s1);
      // dims 16q .. 16q + 15: half q / 4, 16-byte chunks 2 (q % 4) and 2 (q % 4) + 1
      const uint32_t ra = buf + (uint32_t)(q >> 2) * kHalfBytes + (uint32_t)row[u] * 128;
      const uint32_t sw = (uint32_t)(row[u] & 7), c0 = 2u * (uint32_t)(q & 3);
      uint32_t o[4];
      if (fold) cvt_i8x8(w[u].x, w[u].y, s2, true, o); else cvt_i8_f16x8(w[u].x, w[u].y, o);
      st_shared_v4(ra + ((c0 ^ sw) << 4), o[0], o[1], o[2], o[3]);
      if (fold) cvt_i8x8(w[u].z, w[u].w, s2, true, o); else cvt_i8_f16x8(w[u].z, w[u].w, o);
      st_shared_v4(ra + (((c0 + 1) ^ sw) << 4), o[0], o[1], o[2], o[3]);
    }
  }
}

// int4 in place: staged code rows are 64 bytes, so a bf16 row of the upper half
// overlaps two code rows of other slots.  Every loader thread first reads all its
// chunks (chunk ch = 32 codes of row ch / 4), the 96 threads meet at a named barrier,
// then all write (keys to exact f16, values to bf16(code * scale)).  sv holds the
// value scales of the chunks' rows (pairs).
constexpr int kI4Per = (BN * 4 + kConvThreads - 1) / kConvThreads;  // 512 chunks
constexpr int kConvBar = 3;  // named barrier of the loader threads (0: CTA, 1-2: softmax)
__device__ __forceinline__ void convert_i4_read(uint32_t buf, int nv, int ct, uint4 (&w)[kI4Per]) {
#pragma unroll
  for (int r = 0; r < kI4Per; ++r) {
    const int ch = ct + kConvThreads * r;
    w[r] = make_uint4(0u, 0u, 0u, 0u);
    if (ch < BN * 4 && (ch >> 2) < nv) w[r] = ld_shared_v4(buf + kStageOff + ch * 16);
  }
}
// (after every loader thread has read its chunks and met at the named barrier)
__device__ __forceinline__ void convert_i4_write(uint32_t buf, const __half2 (&sv)[(kI4Per + 1) / 2],
                                                 bool fold, int ct, const uint4 (&w)[kI4Per]) {
#pragma unroll
  for (int r = 0; r < kI4Per; ++r) {
    const int ch = ct + kConvThreads * r;
    if (ch >= BN * 4) continue;
    const int j = ch >> 2, q = ch & 3;
    const float sc = fold ? ((r & 1) ? __high2float(sv[r / 2]) : __low2float(sv[r / 2])) : 0.f;
    const float2 s2 = make_float2(sc, sc);
    // dims 32q .. 32q + 31: half q / 2, 16-byte chunks 4 (q % 2) .. 4 (q % 2) + 3
    const uint32_t ra = buf + (uint32_t)(q >> 1) * kHalfBytes + (uint32_t)j * 128;
    const uint32_t sw = (uint32_t)(j & 7), c0 = 4u * (uint32_t)(q & 1);
    const uint32_t ws[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      uint32_t o[4];
      if (fold) cvt_i4x8(ws[m], s2, true, o); else cvt_i4_f16x8(ws[m], o);
      st_shared_v4(ra + (((c0 + m) ^ sw) << 4), o[0], o[1], o[2], o[3]);
    }
  }
}

// The loaders' sequence of tiles: phase A keys 0 .. n_kt - 1 (buffers K0, K1, V0, V1
// in turn), then phase B K(0), K(1), V(0), K(2), V(1), ..., V(n_kt - 1): the order in
// which the MMA issuer consumes them.  use = how many earlier tiles went to the buffer
// (its LOADED barrier phase).
struct LoadItem {
  int kind;  // 0: phase A key tile, 1: phase B key tile, 2: value tile
  int kt, buf, use;
};
__device__ __forceinline__ int uses_a(int b, int n_kt) {
  return b < n_kt ? (n_kt - 1 - b) / kStagesA + 1 : 0;
}
__device__ __forceinline__ LoadItem load_item(int e, int n_kt) {
  LoadItem x;
  if (e < n_kt) {
    x.kind = 0;
    x.kt = e;
    x.buf = e % kStagesA;
    x.use = e / kStagesA;
    return x;
  }
  const int r = e - n_kt;
  if (r == 0) {
    x.kind = 1;
    x.kt = 0;
  } else if (r & 1) {
    const int s = (r + 1) >> 1;
    x.kind = s < n_kt ? 1 : 2;
    x.kt = s < n_kt ? s : n_kt - 1;
  } else {
    x.kind = 2;
    x.kt = (r >> 1) - 1;
  }
  const int b = x.kt & 1;
  x.buf = x.kind == 1 ? b : 2 + b;
  x.use = uses_a(x.buf, n_kt) + (x.kt >> 1);
  return x;
}

// Key scales times the raw logits of one row (phase A, quantized caches).
template <int N>
__device__ __forceinline__ void scale_row(uint32_t (&x)[N], const float *ks) {
#pragma unroll
  for (int e = 0; e < N; e += 4) {
    const float4 k4 = *reinterpret_cast<const float4 *>(ks + e);
    const float2 a = mul2(make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])),
                          make_float2(k4.x, k4.y));
    const float2 b = mul2(make_float2(__uint_as_float(x[e + 2]), __uint_as_float(x[e + 3])),
                          make_float2(k4.z, k4.w));
    x[e] = __float_as_uint(a.x);
    x[e + 1] = __float_as_uint(a.y);
    x[e + 2] = __float_as_uint(b.x);
    x[e + 3] = __float_as_uint(b.y);
  }
}

template <int KV>
__global__ void __launch_bounds__(threads_of<KV>(), 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap q_map,
                   const __grid_constant__ CUtensorMap k_map,
                   const __grid_constant__ CUtensorMap v_map, const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // the swizzled operand tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicExch(p.status, H2OKV_ERR_CUDA);
    return;
  }
  int32_t *tp_s = reinterpret_cast<int32_t *>(smem + OFF_TP);
  float *lse_s = reinterpret_cast<float *>(smem + OFF_LSE);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + OFF_TMEM);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // work: query tiles 2c and 2c+1 of group bg, in (head, row tile) order
  const int bg = blockIdx.x / p.ctas_per_group;
  const int c = blockIdx.x - bg * p.ctas_per_group;
  const int b = bg / p.Hk, g = bg - b * p.Hk;
  const int n_qt = p.q_g * p.tiles;
  const int qa = 2 * c, qb = 2 * c + 1;
  const bool has_b = qb < n_qt;
  const int hl_a = qa / p.tiles, t_a = qa - hl_a * p.tiles;
  const int hl_b = has_b ? qb / p.tiles : hl_a, t_b = has_b ? qb - hl_b * p.tiles : t_a;
  const int bhq_a = b * p.Hq + g * p.q_g + hl_a, bhq_b = b * p.Hq + g * p.q_g + hl_b;
  const int i0_a = t_a * BM, i0_b = t_b * BM;
  const int n_kt = p.n_kt;
  const uint64_t lim = p.timeout_ns;

  const int nwg = has_b ? 2 : 1;  // softmax warpgroups with a query tile
  // tile-full barriers: one TMA producer (bf16) or the three loader warps (quantized)
  constexpr uint32_t kFullCount = KV == H2OKV_BF16 ? 1 : kConvThreads / 32;
  if (threadIdx.x == 0) {
    mbar_init(&bar[B_Q], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[B_KFULL0 + i], kFullCount);
      mbar_init(&bar[B_KEMPTY0 + i], 1 + 4 * nwg);  // MMA commit + softmax warps (token positions)
      mbar_init(&bar[B_VFULL0 + i], kFullCount);
      mbar_init(&bar[B_VEMPTY0 + i], 1);
      mbar_init(&bar[B_SFULL0 + i], 1);
      mbar_init(&bar[B_SFREE0 + i], 4 * nwg);
    }
    mbar_init(&bar[B_AFREE], 4 * nwg);
    mbar_init(&bar[B_TFULLA], 1);
    mbar_init(&bar[B_TFULLB], 1);
    mbar_init(&bar[B_TFREEA], 4);
    mbar_init(&bar[B_TFREEB], 4);
    mbar_init(&bar[B_PFULLA], 4);
    mbar_init(&bar[B_PFULLB], 4);
    mbar_init(&bar[B_PFREEA], 1);
    mbar_init(&bar[B_PFREEB], 1);
    mbar_init(&bar[B_OFULL], 1);
    mbar_init(&bar[B_DRAIN], 1);
    mbar_init(&bar[B_VGO], 1);
    for (int i = 0; i < kStagesA; ++i) {
      mbar_init(&bar[B_AFULL0 + i], kFullCount);
      mbar_init(&bar[B_AEMPTY0 + i], 1 + 4 * nwg);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&bar[B_LOADED0 + i], 1);
    mbar_init(&bar[B_QREADY], kConvThreads / 32);
    tmem_s[1] = 0;  // loader abort flag (quantized caches)
    tmem_s[2] = 0;  // largest |q| of query tile a / b (float bits; quantized caches)
    tmem_s[3] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_s, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&q_map);
    if (KV == H2OKV_BF16) {
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_s;
  bool aborted = false;
  // logits Q K^T: bf16 operands, or f16 for quantized caches (exact integer keys)
  constexpr uint32_t kIdescS = KV == H2OKV_BF16 ? IDESC_K_MAJOR : IDESC_K_MAJOR_F16;

  if (warp < 4 || warp >= 12) {
  reg_dealloc<KV == H2OKV_BF16 ? kCtrlRegs : kCtrlRegsQ>();
  if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t qa_addr = sbase + OFF_QA, qb_addr = sbase + OFF_QB, p_addr = sbase + OFF_P;
      if (!mbar_wait(&bar[KV == H2OKV_BF16 ? B_Q : B_QREADY], 0, lim)) fail(p, aborted);
      tc_fence_after();
      // phase A: S_a, S_b = Q_a K^T, Q_b K^T into the column pair of the tile parity
      for (int kt = 0; kt < n_kt && !aborted; ++kt) {
        const int a = kt % kStagesA, u = kt & 1;
        if (!mbar_wait(&bar[B_AFULL0 + a], (kt / kStagesA) & 1, lim)) { fail(p, aborted); break; }
        if (kt >= 2 && !mbar_wait(&bar[B_SFREE0 + u], ((kt >> 1) - 1) & 1, lim)) {
          fail(p, aborted);
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = sbase + slot_a(a);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16_ss(tmem + u * 256, kmajor_desc(qa_addr, ks), kmajor_desc(k_addr, ks),
                      kIdescS, ks > 0);
        if (has_b) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_bf16_ss(tmem + u * 256 + 128, kmajor_desc(qb_addr, ks), kmajor_desc(k_addr, ks),
                        kIdescS, ks > 0);
        }
        mma_commit(&bar[B_SFULL0 + u]);
        mma_commit(&bar[B_AEMPTY0 + a]);
      }
      mma_commit(&bar[B_VGO]);  // phase A K tiles in slots V0 / V1 no longer read
      // every phase A TMEM read is done before phase B reuses the columns
      if (!aborted && !mbar_wait(&bar[B_AFREE], 0, lim)) fail(p, aborted);
      tc_fence_after();
      // phase B.  S^T_x(kt) = K(kt) Q_x^T into columns 0 (a) / 128 (b);
      // O_x += P_x(kt) V(kt) into columns 256 (a) / 384 (b).
      auto issue_st = [&](int kt, bool tile_b) -> bool {
        const int s = kt & 1;
        if (!tile_b && !mbar_wait(&bar[B_KFULL0 + s], (kt >> 1) & 1, lim)) return false;
        if (kt >= 1 && !mbar_wait(&bar[tile_b ? B_TFREEB : B_TFREEA], (kt - 1) & 1, lim))
          return false;
        tc_fence_after();
        const uint32_t k_addr = sbase + (s ? OFF_K1 : OFF_K0);
        const uint32_t q_addr = tile_b ? qb_addr : qa_addr;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16_ss(tmem + (tile_b ? 128 : 0), kmajor_desc(k_addr, ks), kmajor_desc(q_addr, ks),
                      kIdescS, ks > 0);
        mma_commit(&bar[tile_b ? B_TFULLB : B_TFULLA]);
        if (tile_b || !has_b) mma_commit(&bar[B_KEMPTY0 + s]);  // K(kt) no longer read
        return true;
      };
      auto issue_pv = [&](int kt, bool tile_b) -> bool {
        if (!mbar_wait(&bar[tile_b ? B_PFULLB : B_PFULLA], kt & 1, lim)) return false;
        if (!tile_b && !mbar_wait(&bar[B_VFULL0 + (kt & 1)], (kt >> 1) & 1, lim)) return false;
        tc_fence_after();
        const uint32_t v_addr = sbase + ((kt & 1) ? OFF_V1 : OFF_V0);
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_bf16_ss(tmem + (tile_b ? 384 : 256), mnmajor_desc(p_addr, ks),
                      mnmajor_desc(v_addr, ks), IDESC_PV, (kt > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bar[tile_b ? B_PFREEB : B_PFREEA]);
        if (tile_b || !has_b) mma_commit(&bar[B_VEMPTY0 + (kt & 1)]);  // V(kt) no longer read
        return true;
      };
      if (!aborted && !issue_st(0, false)) fail(p, aborted);
      if (!aborted && has_b && !issue_st(0, true)) fail(p, aborted);
      // S^T of the next tile is issued as soon as the softmax warps have read the
      // current one out of TMEM (long before their P is ready), then the P V
      // products of the current tile.
      for (int kt = 0; kt < n_kt && !aborted; ++kt) {
        if (kt + 1 < n_kt && !issue_st(kt + 1, false)) { fail(p, aborted); break; }
        if (kt + 1 < n_kt && has_b && !issue_st(kt + 1, true)) { fail(p, aborted); break; }
        if (!issue_pv(kt, false)) { fail(p, aborted); break; }
        if (has_b && !issue_pv(kt, true)) { fail(p, aborted); break; }
      }
      mma_commit(&bar[B_OFULL]);
      // drain: every MMA issued by this thread completes before TMEM is freed
      mma_commit(&bar[B_DRAIN]);
      mbar_wait(&bar[B_DRAIN], 0, 4000000000ull);
    }
    __syncwarp();
  } else if constexpr (KV == H2OKV_BF16) {
  if (warp == 0) {
    // ------------------------------------------------- producer of Q, K and token positions
    if (lane == 0) {
      mbar_expect_tx(&bar[B_Q], has_b ? 2 * kTileBytes : kTileBytes);
      tma_load_3d(smem + OFF_QA, &q_map, &bar[B_Q], 0, i0_a, bhq_a);
      tma_load_3d(smem + OFF_QA + kHalfBytes, &q_map, &bar[B_Q], 64, i0_a, bhq_a);
      if (has_b) {
        tma_load_3d(smem + OFF_QB, &q_map, &bar[B_Q], 0, i0_b, bhq_b);
        tma_load_3d(smem + OFF_QB + kHalfBytes, &q_map, &bar[B_Q], 64, i0_b, bhq_b);
      }
      mbar_arrive(&bar[B_Q]);
    }
    const int32_t *tpg = p.token_pos + (size_t)bg * p.N_C;
    int issued_a = 0, issued_b = 0;
    for (int it = 0; it < 2 * n_kt && !aborted; ++it) {
      const bool phB = it >= n_kt;
      const int kt = phB ? it - n_kt : it;
      int stage;
      uint64_t *full;
      uint8_t *kdst;
      int32_t *tdst;
      if (!phB) {  // phase A: four stages
        stage = kt % kStagesA;
        const int n = kt / kStagesA;
        if (n > 0 && !warp_wait(&bar[B_AEMPTY0 + stage], (n - 1) & 1, lim)) { fail(p, aborted); break; }
        full = &bar[B_AFULL0 + stage];
        kdst = smem + slot_a(stage);
        tdst = reinterpret_cast<int32_t *>(smem + OFF_P) + stage * BN;
      } else {  // phase B: slots K0 / K1 after their last phase A use
        stage = kt & 1;
        bool ok;
        if (kt < 2) {
          const int lu = last_use_a(stage, n_kt);
          ok = lu < 0 || warp_wait(&bar[B_AEMPTY0 + stage], (lu / kStagesA) & 1, lim);
        } else {
          ok = warp_wait(&bar[B_KEMPTY0 + stage], ((kt >> 1) - 1) & 1, lim);
        }
        if (!ok) { fail(p, aborted); break; }
        full = &bar[B_KFULL0 + stage];
        kdst = smem + (stage ? OFF_K1 : OFF_K0);
        tdst = tp_s + stage * BN;
      }
      const int nv = min(BN, p.N_C - kt * BN);  // slots of this tile inside the cache
      if (lane == 0) {
        mbar_expect_tx(full, kTileBytes);
        tma_load_3d(kdst, &k_map, full, 0, kt * BN, bg);
        tma_load_3d(kdst + kHalfBytes, &k_map, full, 64, kt * BN, bg);
        // bring the K tiles kPrefetch loads ahead into L2
        const int ahead = it + kPrefetch;
        if (ahead < 2 * n_kt) {
          const int kta = ahead >= n_kt ? ahead - n_kt : ahead;
          tma_prefetch_l2_3d(&k_map, 0, kta * BN, bg);
          tma_prefetch_l2_3d(&k_map, 64, kta * BN, bg);
        }
      }
      // position of each slot's token relative to the chunk start, as a float:
      // row i of the chunk sees the slot iff rel <= i (empty / outside slots: 2^20)
#pragma unroll
      for (int e = lane; e < BN; e += 32) {
        const int64_t t = e < nv ? (int64_t)tpg[kt * BN + e] : (int64_t)kEmptyPos;
        const int64_t rel = t - (int64_t)p.P;
        tdst[e] = __float_as_int((float)(rel < -1 ? -1 : (rel > kRelFar ? kRelFar : rel)));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(full);
      if (phB) issued_b = kt + 1; else issued_a = kt + 1;
    }
    // drain: the last issued loads of both rings must land before exit
    if (lane == 0) {
      mbar_wait(&bar[B_Q], 0, 4000000000ull);
      for (int kt = issued_a - 1; kt >= 0 && kt >= issued_a - kStagesA; --kt)
        mbar_wait(&bar[B_AFULL0 + kt % kStagesA], (kt / kStagesA) & 1, 4000000000ull);
      for (int kt = issued_b - 1; kt >= 0 && kt >= issued_b - 2; --kt)
        mbar_wait(&bar[B_KFULL0 + (kt & 1)], (kt >> 1) & 1, 4000000000ull);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------------ producer of V
    if (lane == 0) {
      int v_issued = 0;
      for (int kt = 0; kt < n_kt && !aborted; ++kt) {
        const int vs = kt & 1, vn = kt >> 1;
        bool ok;
        if (vn == 0) {  // slots V0 / V1 serve as phase A K stages 2 / 3 until every phase A MMA is done
          ok = mbar_wait(&bar[B_VGO], 0, lim);
        } else {
          ok = mbar_wait(&bar[B_VEMPTY0 + vs], (vn - 1) & 1, lim);
        }
        if (!ok) {
          fail(p, aborted);
          break;
        }
        uint8_t *vdst = smem + (vs ? OFF_V1 : OFF_V0);
        mbar_expect_tx(&bar[B_VFULL0 + vs], kTileBytes);
        tma_load_3d(vdst, &v_map, &bar[B_VFULL0 + vs], 0, kt * BN, bg);
        tma_load_3d(vdst + kHalfBytes, &v_map, &bar[B_VFULL0 + vs], 64, kt * BN, bg);
        mbar_arrive(&bar[B_VFULL0 + vs]);
        if (kt + kPrefetch < n_kt) {
          tma_prefetch_l2_3d(&v_map, 0, (kt + kPrefetch) * BN, bg);
          tma_prefetch_l2_3d(&v_map, 64, (kt + kPrefetch) * BN, bg);
        }
        v_issued = kt + 1;
      }
      for (int kt = v_issued - 1; kt >= 0 && kt >= v_issued - 2; --kt)
        mbar_wait(&bar[B_VFULL0 + (kt & 1)], (kt >> 1) & 1, 4000000000ull);
    }
    __syncwarp();
  }
  } else {
    // --------------------------- loaders of quantized tiles (warps 0, 2, 3: 96 threads)
    const int w3 = warp == 0 ? 0 : (warp < 4 ? warp - 1 : warp - 9);  // 0 .. kLoaderWarps - 1
    const int ct = 32 * w3 + lane;
    if (warp == 0 && lane == 0) {
      mbar_expect_tx(&bar[B_Q], has_b ? 2 * kTileBytes : kTileBytes);
      tma_load_3d(smem + OFF_QA, &q_map, &bar[B_Q], 0, i0_a, bhq_a);
      tma_load_3d(smem + OFF_QA + kHalfBytes, &q_map, &bar[B_Q], 64, i0_a, bhq_a);
      if (has_b) {
        tma_load_3d(smem + OFF_QB, &q_map, &bar[B_Q], 0, i0_b, bhq_b);
        tma_load_3d(smem + OFF_QB + kHalfBytes, &q_map, &bar[B_Q], 64, i0_b, bhq_b);
      }
      mbar_arrive(&bar[B_Q]);
    }
    constexpr int RB = QTile<KV>::kRowBytes;
    const int32_t *tpg = p.token_pos + (size_t)bg * p.N_C;
    const uint8_t *kg = p.kq + (size_t)bg * p.N_C * RB;
    const uint8_t *vg = p.vq + (size_t)bg * p.N_C * RB;
    const __half *ksg = p.ksc + (size_t)bg * p.N_C;
    const __half *vsg = p.vsc + (size_t)bg * p.N_C;
    volatile uint32_t *abort_flag = tmem_s + 1;
    __half *ksb = reinterpret_cast<__half *>(smem + OFF_KSB);
    // The query tiles become f16 once: tile t is divided by 2^e_t so that its largest
    // |q| lies in [2^14, 2^15) (the softmax warps multiply the logit scale by 2^e_t);
    // for int4 caches the 8 elements of every 16-byte chunk take the keys' order.
    {
      const bool qok = warp_wait(&bar[B_Q], 0, lim);
      if (!qok) {
        fail(p, aborted);
        if (lane == 0) *abort_flag = 1u;
      }
      const int nch = (has_b ? 2 : 1) * (int)(kTileBytes / 16);
      uint32_t mx0 = 0u, mx1 = 0u;  // largest |bf16| bit pattern of tile a / b
      if (qok) {
        for (int ch = ct; ch < nch; ch += kConvThreads) {
          const uint4 v = ld_shared_v4(sbase + OFF_QA + (uint32_t)ch * 16);
          const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
          uint32_t m = 0u;
#pragma unroll
          for (int i = 0; i < 4; ++i) m = max(m, max(ws[i] & 0x7FFFu, (ws[i] >> 16) & 0x7FFFu));
          if (ch < (int)(kTileBytes / 16)) mx0 = max(mx0, m); else mx1 = max(mx1, m);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mx0 = max(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = max(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      if (lane == 0) {
        atomicMax(const_cast<uint32_t *>(tmem_s) + 2, mx0 << 16);
        atomicMax(const_cast<uint32_t *>(tmem_s) + 3, mx1 << 16);
      }
      named_bar_sync(kConvBar, kConvThreads);
      if (*abort_flag) {
        aborted = true;
      } else {
        const float f0 = exp2i(-q_exponent(tmem_s[2])), f1 = exp2i(-q_exponent(tmem_s[3]));
        for (int ch = ct; ch < nch; ch += kConvThreads) {
          const uint32_t addr = sbase + OFF_QA + (uint32_t)ch * 16;
          const uint4 v = ld_shared_v4(addr);
          const float f = ch < (int)(kTileBytes / 16) ? f0 : f1;
          const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
          float e[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            e[2 * i] = __uint_as_float(ws[i] << 16) * f;
            e[2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u) * f;
          }
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int lo = KV == H2OKV_I4 ? i : 2 * i, hi = KV == H2OKV_I4 ? i + 4 : 2 * i + 1;
            const __half2 h = __floats2half2_rn(e[lo], e[hi]);
            o[i] = *reinterpret_cast<const uint32_t *>(&h);
          }
          st_shared_v4(addr, o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_QREADY]);
      }
    }
    const int E = aborted ? 0 : 3 * n_kt;
    // The buffer a tile goes to is free once the previous tile in it has been consumed:
    // the same conditions the TMA producers of a bf16 cache wait for.
    auto free_cond = [&](const LoadItem &x, uint64_t *&fb, uint32_t &par) -> bool {
      if (x.kind == 0) {
        const int n = x.kt / kStagesA;
        if (n == 0) return false;
        fb = &bar[B_AEMPTY0 + x.buf];
        par = (uint32_t)(n - 1) & 1u;
      } else if (x.kind == 1) {
        const int st = x.kt & 1;
        if (x.kt < 2) {
          const int lu = last_use_a(st, n_kt);
          if (lu < 0) return false;
          fb = &bar[B_AEMPTY0 + st];
          par = (uint32_t)(lu / kStagesA) & 1u;
        } else {
          fb = &bar[B_KEMPTY0 + st];
          par = (uint32_t)((x.kt >> 1) - 1) & 1u;
        }
      } else {
        const int vn = x.kt >> 1;
        fb = vn == 0 ? &bar[B_VGO] : &bar[B_VEMPTY0 + (x.kt & 1)];
        par = vn == 0 ? 0u : (uint32_t)(vn - 1) & 1u;
      }
      return true;
    };
    // per tile: slot positions relative to the chunk and key scales (threads ct and
    // ct + 96 of the tile), and value scales of this lane's rows
    struct Meta {
      float rel[2];
      __half2 ks;
      __half2 sv[(kI8Passes + 2) / 2];
    };
    auto load_meta = [&](int e) -> Meta {
      const LoadItem x = load_item(e, n_kt);
      const int slot0 = x.kt * BN, nv = min(BN, p.N_C - slot0);
      Meta m;
      __half kh[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int e2 = ct + kConvThreads * i;
        m.rel[i] = (float)kRelFar;
        kh[i] = __float2half(0.f);
        if (x.kind != 2 && e2 < BN && e2 < nv) {
          const int64_t rel = (int64_t)tpg[slot0 + e2] - (int64_t)p.P;
          m.rel[i] = (float)(rel < -1 ? -1 : (rel > kRelFar ? kRelFar : rel));
          kh[i] = ksg[slot0 + e2];
        }
      }
      m.ks = __halves2half2(kh[0], kh[1]);
      __half sh[2 * ((kI8Passes + 2) / 2)];
#pragma unroll
      for (int i = 0; i < 2 * ((kI8Passes + 2) / 2); ++i) {
        int row = BN;
        if (KV == H2OKV_I8)
          row = i < kI8Passes ? 4 * (w3 + kLoaderWarps * i) + (lane >> 3) : BN;
        else
          row = i < kI4Per ? (ct + kConvThreads * i) >> 2 : BN;
        sh[i] = (x.kind == 2 && row < nv) ? vsg[slot0 + row] : __float2half(0.f);
      }
#pragma unroll
      for (int i = 0; i < (kI8Passes + 2) / 2; ++i) m.sv[i] = __halves2half2(sh[2 * i], sh[2 * i + 1]);
      return m;
    };
    Meta meta = E > 0 ? load_meta(0) : Meta{};
    int issued = 0;
    uint32_t last_par = 0;  // per buffer b: bit 2b = a copy was issued, bit 2b + 1 = its parity
    for (int e = 0; e < E; ++e) {
      const LoadItem x = load_item(e, n_kt);
      const int slot0 = x.kt * BN, nv = min(BN, p.N_C - slot0);
      // one thread keeps the copies going: item e (waiting for its buffer) and, while
      // their buffers are already free, the next two
      if (ct == 0 && !aborted) {
        while (issued < E && issued <= e + 2) {
          const LoadItem y = load_item(issued, n_kt);
          uint64_t *fb = nullptr;
          uint32_t par = 0;
          if (free_cond(y, fb, par)) {
            const bool ready = issued == e ? mbar_wait(fb, par, lim) : mbar_test(fb, par);
            if (!ready) {
              if (issued == e) fail(p, aborted);
              break;
            }
          }
          const int y0 = y.kt * BN, ynv = min(BN, p.N_C - y0);
          uint64_t *lb = &bar[B_LOADED0 + y.buf];
          mbar_expect_tx(lb, (uint32_t)(ynv * RB));
          bulk_load(smem + slot_a(y.buf) + kStageOff, (y.kind == 2 ? vg : kg) + (size_t)y0 * RB,
                    (uint32_t)(ynv * RB), lb);
          mbar_arrive(lb);
          last_par = (last_par & ~(3u << (2 * y.buf))) |
                     ((1u | (((uint32_t)y.use & 1u) << 1)) << (2 * y.buf));
          ++issued;
        }
        // bring a later tile's codes, scales and positions into L2
        const int ep = e + 6;
        if (ep < E) {
          const LoadItem z = load_item(ep, n_kt);
          const int z0 = z.kt * BN, znv = min(BN, p.N_C - z0);
          bulk_prefetch_l2((z.kind == 2 ? vg : kg) + (size_t)z0 * RB, (uint32_t)(znv * RB));
          const __half *sp = (z.kind == 2 ? vsg : ksg) + z0;
          if (znv == BN && (reinterpret_cast<uintptr_t>(sp) & 15u) == 0) bulk_prefetch_l2(sp, BN * 2);
          if (z.kind != 2 && znv == BN && (reinterpret_cast<uintptr_t>(tpg + z0) & 15u) == 0)
            bulk_prefetch_l2(tpg + z0, BN * 4);
        }
      }
      const Meta cur = meta;
      // the codes have landed (and the buffer's previous tile was consumed)
      bool ok = !aborted && warp_wait(&bar[B_LOADED0 + x.buf], (uint32_t)x.use & 1u, lim);
      if (!ok) fail(p, aborted);
      uint4 w4[kI4Per];
      if constexpr (KV == H2OKV_I4) {
        // in place: every staged chunk is read before any is overwritten; the loaders
        // meet at a named barrier (and leave the loop together after a failed wait)
        if (!ok && lane == 0) *abort_flag = 1u;
        if (ok) convert_i4_read(sbase + slot_a(x.buf), nv, ct, w4);
        named_bar_sync(kConvBar, kConvThreads);
        if (*abort_flag) {
          aborted = true;
          break;
        }
      } else {
        if (!ok) break;
      }
      // the next tile's positions and scales are read while this one is converted
      if (e + 1 < E) meta = load_meta(e + 1);
      float relv[2], ksv[2];
      __half ksh[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        relv[i] = cur.rel[i];
        ksh[i] = i ? __high2half(cur.ks) : __low2half(cur.ks);
        ksv[i] = __half2float(ksh[i]);
      }
      float sv8[kI8Passes + 1];
#pragma unroll
      for (int i = 0; i <= kI8Passes; ++i)
        sv8[i] = (i & 1) ? __high2float(cur.sv[i / 2]) : __low2float(cur.sv[i / 2]);
      __half2 sv4[(kI4Per + 1) / 2];
#pragma unroll
      for (int r = 0; r < (kI4Per + 1) / 2; ++r) sv4[r] = cur.sv[r];
      if (x.kind == 0) {
        float *rd = reinterpret_cast<float *>(smem + OFF_REL_A) + x.buf * BN;
        float *kd = reinterpret_cast<float *>(smem + OFF_KS_A) + x.buf * BN;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int e2 = ct + kConvThreads * i;
          if (e2 < BN) {
            rd[e2] = relv[i];
            kd[e2] = ksv[i];
          }
        }
      } else if (x.kind == 1) {
        float *rd = reinterpret_cast<float *>(tp_s) + x.buf * BN;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int e2 = ct + kConvThreads * i;
          if (e2 < BN) {
            rd[e2] = relv[i];
            ksb[x.buf * BN + e2] = ksh[i];
          }
        }
      }
      const uint32_t buf = sbase + slot_a(x.buf);
      if constexpr (KV == H2OKV_I8)
        convert_i8(buf, nv, sv8, x.kind == 2, w3, lane);
      else
        convert_i4_write(buf, sv4, x.kind == 2, ct, w4);
      // the stores of this warp reach the async proxy, then one arrival per warp
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0)
        mbar_arrive(x.kind == 0 ? &bar[B_AFULL0 + x.buf]
                                : (x.kind == 1 ? &bar[B_KFULL0 + x.buf] : &bar[B_VFULL0 + x.buf - 2]));
    }
    // drain: the Q copy and the last copy into each buffer must land before exit
    if (ct == 0) {
      mbar_wait(&bar[B_Q], 0, 4000000000ull);
      for (int b2 = 0; b2 < 4; ++b2)
        if ((last_par >> (2 * b2)) & 1u)
          mbar_wait(&bar[B_LOADED0 + b2], (last_par >> (2 * b2 + 1)) & 1u, 4000000000ull);
    }
    __syncwarp();
  }
  } else {
  reg_alloc<KV == H2OKV_BF16 ? kSoftRegs : kSoftRegsQ>();
  if (warp < 8 || has_b) {
    // -------------------------------------------- softmax / sums, one warpgroup per query tile
    const int wg = (warp - 4) >> 2;  // 0: tile a, 1: tile b
    const int st = threadIdx.x - 128 * (1 + wg);  // row (phase A) or slot (phase B) in the tile
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    float c2 = p.scale2;
    if constexpr (KV != H2OKV_BF16) {
      // the query tile was divided by 2^e before it became f16
      if (!warp_wait(&bar[B_QREADY], 0, lim)) fail(p, aborted);
      c2 *= exp2i(q_exponent(tmem_s[2 + wg]));
    }
    const int i0 = wg ? i0_b : i0_a, bhq = wg ? bhq_b : bhq_a, t = wg ? t_b : t_a;
    float m = -INFINITY, l = 0.f;
    const float mbias = kMaskBias / c2;
    uint32_t x[BN];
    for (int kt = 0; kt < n_kt && !aborted; ++kt) {
      const int u = kt & 1, a = kt % kStagesA;
      if (!warp_wait(&bar[B_SFULL0 + u], (kt >> 1) & 1, lim)) { fail(p, aborted); break; }
      if (!warp_wait(&bar[B_AFULL0 + a], (kt / kStagesA) & 1, lim)) { fail(p, aborted); break; }
      tc_fence_after();
      const float *rela = reinterpret_cast<const float *>(smem + OFF_P) + a * BN;
      // any slot of this tile invisible to some row of this query tile?
      const float rv = fmax3(fmaxf(rela[lane], rela[lane + 32]), rela[lane + 64], rela[lane + 96]);
      const bool masked = __any_sync(0xffffffffu, rv > (float)i0);
      const uint32_t sa = tmem + lane_base + u * 256 + wg * 128;
      tmem_ld32(sa, *reinterpret_cast<uint32_t(*)[32]>(x));
      tmem_ld32(sa + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
      tmem_ld32(sa + 64, *reinterpret_cast<uint32_t(*)[32]>(x + 64));
      tmem_ld32(sa + 96, *reinterpret_cast<uint32_t(*)[32]>(x + 96));
      tmem_wait_ld();
      if constexpr (KV != H2OKV_BF16)
        scale_row<BN>(x, reinterpret_cast<const float *>(smem + OFF_KS_A) + a * BN);
      if (masked) row_mask<BN>(x, rela, (float)(i0 + st), mbias);
      // S buffer and K stage (with its token positions) are free once read
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[B_SFREE0 + u]);
        mbar_arrive(&bar[B_AEMPTY0 + a]);
      }
      row_update<BN>(x, c2, m, l);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar[B_AFREE]);
    // masked logits sit 2^30 below the visible ones: a row whose maximum is that
    // low sees no slot (lse = -inf, no weight, y = 0)
    const bool seen = l > 0.f && m > -0.5f * kMaskBias;
    const float lse2 = seen ? m + lg2(l) : -INFINITY;
    float *lse_t = lse_s + wg * BM;  // holds -lse2 of the tile's rows
    lse_t[st] = seen ? -lse2 : -kMaskBias;
    if (p.lse_out && i0 + st < p.S)
      p.lse_out[(size_t)bhq * p.S + i0 + st] = lse2 * 0.69314718055994531f;
    named_bar_sync(1 + wg, 128);

    // phase B
    const int rmax = min(BM, p.S - i0);
    float *pw = p.part_w + ((size_t)bhq * p.tiles + t) * p.N_C;
    const uint32_t p_row = sbase + OFF_P + (st >> 3) * 1024 + (st & 7) * 128;
    uint32_t pk[BM / 2];
    for (int kt = 0; kt < n_kt && !aborted; ++kt) {
      const int s = kt & 1;
      const int j = kt * BN + st;
      if (!warp_wait(&bar[wg ? B_TFULLB : B_TFULLA], kt & 1, lim)) { fail(p, aborted); break; }
      if (!warp_wait(&bar[B_KFULL0 + s], (kt >> 1) & 1, lim)) { fail(p, aborted); break; }
      tc_fence_after();
      const float relj = __int_as_float(tp_s[s * BN + st]);
      // quantized caches: the slot's key scale joins the logit scale
      const float c2j = KV == H2OKV_BF16
                            ? c2
                            : c2 * __half2float(reinterpret_cast<const __half *>(smem + OFF_KSB)[s * BN + st]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_KEMPTY0 + s]);
      // visible rows r of this tile: relj <= i0 + r, r < rmax
      const float rmf = fminf(fmaxf(relj - (float)i0, 0.f), (float)BM);
      const int rmin = (int)rmf;
      const bool full = __all_sync(0xffffffffu, rmin == 0 && rmax == BM);
      uint32_t r[BM];
      tmem_ld128(tmem + lane_base + wg * 128, r);
      // S^T buffer is free once read: the next tile's logits can be computed meanwhile
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[wg ? B_TFREEB : B_TFREEA]);
      const float cs = slot_probs(r, lse_t, c2j, rmin, rmax, full, pk);
      // the single P buffer goes a(kt) -> b(kt) -> a(kt+1): wait for the previous reader
      bool ok = true;
      if (wg == 1)
        ok = warp_wait(&bar[B_PFREEA], kt & 1, lim);
      else if (kt > 0)
        ok = warp_wait(&bar[has_b ? B_PFREEB : B_PFREEA], (kt - 1) & 1, lim);
      if (!ok) { fail(p, aborted); break; }
      store_p(p_row, st, pk);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[wg ? B_PFULLB : B_PFULLA]);
      if (j < p.N_C) pw[j] = cs;
    }
    // epilogue: y = O (already normalised)
    if (!aborted && !warp_wait(&bar[B_OFULL], 0, lim)) fail(p, aborted);
    tc_fence_after();
    if (!aborted) {
      const int row_i = i0 + st;
      __nv_bfloat16 *yrow = p.y + ((size_t)bhq * p.S + row_i) * D;
      uint32_t r[32];
#pragma unroll
      for (int cq = 0; cq < 4; ++cq) {
        tmem_ld32(tmem + lane_base + 256 + wg * 128 + cq * 32, r);
        tmem_wait_ld();
        if (row_i < p.S) {
          uint32_t o[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            o[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
          uint4 *dst = reinterpret_cast<uint4 *>(yrow + cq * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
        }
      }
    }
    tc_fence_before();
  }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- bf16 caches, two passes ------------------------------------------------------
// Pass 1 (attn_fwd_kernel): attention of two query tiles against the cache with an
// online softmax.  Per K/V tile: S = Q K^T into TMEM; the softmax warps read their
// row, turn it into probabilities against a running reference maximum and write them
// back over S as bf16 pairs; O += P V then takes P straight from TMEM (the A operand)
// and V from shared memory.  Output: y, and -lse2 of every row for pass 2.
// Pass 2 (scoresum_kernel): the logits again, transposed (S^T = K Q^T, slots on TMEM
// lanes), normalised with the final row LSE and summed over the rows of each slot.
// Neither pass stores P in shared memory; pass 2 reads no V.
constexpr int kStagesF = 3;  // pass 1 K ring
constexpr int kStagesS = 4;  // pass 2 K ring
constexpr float kLazyMax = 8.f;  // the reference maximum moves only when exceeded by 2^8
constexpr uint32_t F_OFF_QA = 0;
constexpr uint32_t F_OFF_QB = kTileBytes;
constexpr uint32_t F_OFF_K = 2 * kTileBytes;                      // [kStagesF] K tiles
constexpr uint32_t F_OFF_V = F_OFF_K + kStagesF * kTileBytes;      // [2] V tiles
constexpr uint32_t F_OFF_REL = F_OFF_V + 2 * kTileBytes;           // float [kStagesF][BN]
// Per K stage, the slots that some row of the CTA may not see (position beyond the
// first row of a query tile): int count, then up to kMaxCand (slot, position) pairs;
// count -1 when there are more (the softmax then masks the whole row).
constexpr int kMaxCand = 16;
constexpr uint32_t F_OFF_CAND = F_OFF_REL + kStagesF * BN * 4;     // [kStagesF][1 + 2 kMaxCand]
constexpr uint32_t kCandWords = 2 + 2 * kMaxCand;                  // count, pad, pairs
// The CTA's segments (pair, first and end K/V tile, partial slot), listed once.
constexpr int kMaxSegF = 15;
constexpr uint32_t F_OFF_SEG = (F_OFF_CAND + kStagesF * kCandWords * 4 + 15) & ~15u;  // int4 [1 + kMaxSegF]
static_assert(F_OFF_SEG % 16 == 0 && F_OFF_CAND % 16 == 0, "pass 1 shared memory alignment");
constexpr uint32_t F_OFF_BAR = F_OFF_SEG + (1 + kMaxSegF) * 16;
enum {
  F_Q = 0,
  F_KFULL0, F_KEMPTY0 = F_KFULL0 + kStagesF,   // K ring (+ slot positions)
  F_VFULL0 = F_KEMPTY0 + kStagesF, F_VEMPTY0 = F_VFULL0 + 2,  // V ring
  F_SFULL0 = F_VEMPTY0 + 2,                    // S of tile a / b written
  F_PFULL0 = F_SFULL0 + 2,                     // P of tile a / b written (O rescaled)
  F_OFULL = F_PFULL0 + 2,                      // a segment's last P V done
  F_OFREE,                                     // a segment's O read out by the softmax warps
  F_QFREE,                                     // a segment's Q tiles no longer read
  F_DRAIN,
  F_END
};
constexpr uint32_t F_OFF_TMEM = F_OFF_BAR + F_END * 8;
// pass 1 register split: the softmax warps hold a row of logits and its packed
// probabilities: 128 x 72 + 256 x 216 = 384 x 168
constexpr int kCtrlRegsF = 72, kSoftRegsF = 216;
static_assert(128 * kCtrlRegsF + 256 * kSoftRegsF == kThreads * kLaunchRegs, "pass 1 register split");
constexpr uint32_t kSmemF = F_OFF_TMEM + 16;
static_assert(kSmemF <= 232448, "pass 1 shared memory budget");
// P (TMEM, K-major) x V (shared memory, MN-major)
constexpr uint32_t IDESC_TS_PV = idesc_bf16_f32(128, 128, false, true);

// Maximum of a row of raw logits (eight independent chains of three-input maxima).
template <int N>
__device__ __forceinline__ float row_max(const uint32_t (&x)[N]) {
  float mx8[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) mx8[q] = fmaxf(__uint_as_float(x[q]), __uint_as_float(x[q + 8]));
#pragma unroll
  for (int e = 16; e < N; e += 16) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      mx8[q] = fmax3(mx8[q], __uint_as_float(x[e + q]), __uint_as_float(x[e + 8 + q]));
  }
  return fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
               fmaxf(mx8[6], mx8[7]));
}

// Probabilities 2^(c2 x - m) of one row of raw logits, packed to bf16 pairs, and
// their sum.
__device__ __forceinline__ float row_probs(const uint32_t (&x)[BN], float c2, float m,
                                           uint32_t (&pk)[BN / 2]) {
  const float2 c2v = make_float2(c2, c2), negm = make_float2(-m, -m);
  float2 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
  for (int e = 0; e < BN; e += 2) {
    const float2 a = fma2(make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])), c2v, negm);
    const float2 v = make_float2(ex2(a.x), ex2(a.y));
    acc[(e >> 1) & 3] = add2(acc[(e >> 1) & 3], v);
    pk[e >> 1] = pack_bf16x2(v.x, v.y);
  }
  const float2 s01 = add2(acc[0], acc[1]), s23 = add2(acc[2], acc[3]);
  const float2 s4 = add2(s01, s23);
  return s4.x + s4.y;
}

// Slot positions of one K tile relative to the chunk start, as floats (row i of the
// chunk sees the slot iff rel <= i; empty or out-of-cache slots: 2^20).  One warp.
__device__ __forceinline__ void tile_positions(float *dst, const int32_t *tpg, int kt, int N_C,
                                               int P, int lane) {
  const int nv = min(BN, N_C - kt * BN);
#pragma unroll
  for (int e = lane; e < BN; e += 32) {
    const int64_t t = e < nv ? (int64_t)tpg[kt * BN + e] : (int64_t)kEmptyPos;
    const int64_t rel = t - (int64_t)P;
    dst[e] = (float)(rel < -1 ? -1 : (rel > kRelFar ? kRelFar : rel));
  }
}

// Pass 2 shared memory: Q_a, Q_b, the K ring, -lse2 of both tiles.
constexpr uint32_t S_OFF_QA = 0;
constexpr uint32_t S_OFF_QB = kTileBytes;
constexpr uint32_t S_OFF_K = 2 * kTileBytes;                   // [kStagesS] K tiles
constexpr uint32_t S_OFF_NLSE = S_OFF_K + kStagesS * kTileBytes;  // float [2 segments][2][BM]
constexpr uint32_t S_OFF_BAR = S_OFF_NLSE + 4 * BM * 4;
enum {
  G_Q = 0,
  G_KFULL0, G_KEMPTY0 = G_KFULL0 + kStagesS,
  G_SFULL0 = G_KEMPTY0 + kStagesS, G_SFREE0 = G_SFULL0 + 2,  // S^T pair, double buffered
  G_QFREE = G_SFREE0 + 2,                                     // Q of a segment no longer read
  G_NL0,                                                      // -lse2 of tile a / b written
  G_DRAIN = G_NL0 + 2,
  G_END
};
constexpr uint32_t S_OFF_TMEM = S_OFF_BAR + G_END * 8;
// pass 2: 4 control warps + 4 softmax warpgroups at 96 registers (640 x 96 = 61440); the
// control warps drop to 64, the softmax warps (half a column of 64 logits at a time)
// rise to 104: 128 x 64 + 512 x 104 = 61440
constexpr int kThreadsS = 640;
constexpr int kLaunchRegsS = 96, kCtrlRegsS = 64, kSoftRegsS = 104;
static_assert(128 * kCtrlRegsS + 512 * kSoftRegsS == kThreadsS * kLaunchRegsS, "pass 2 register split");
constexpr uint32_t kSmemS = S_OFF_TMEM + 16;
static_assert(kSmemS <= 232448, "pass 2 shared memory budget");

// Sum over the rows of one tile of the normalised probabilities of one slot:
// sum_r 2^(c2 s_r - lse2_r) over visible rows r (rmin <= r < rmax).  MASK = false:
// every row visible (rmin = 0, rmax = BM).
template <bool MASK, int N>
__device__ __forceinline__ float slot_colsum(const uint32_t (&r)[N], const float *nlse, float c2,
                                             int rmin, int rmax) {
  const float rminf = (float)rmin;
  const float2 c2v = make_float2(c2, c2);
  float2 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
  for (int e = 0; e < N; e += 2) {
    const float2 nl = *reinterpret_cast<const float2 *>(nlse + e);
    float2 a = fma2(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), c2v, nl);
    if constexpr (MASK) {  // rows before rmin are masked: nm = sat(rmin - row) is 1 there
      const float2 nm = make_float2(fma_sat(rminf, 1.f, -(float)e), fma_sat(rminf, 1.f, -(float)(e + 1)));
      a = fma2(nm, make_float2(-kMaskBias, -kMaskBias), a);
    }
    float2 v = make_float2(ex2(a.x), ex2(a.y));
    if constexpr (MASK) {  // rows past the chunk (last row tile only)
      v.x = e < rmax ? v.x : 0.f;
      v.y = e + 1 < rmax ? v.y : 0.f;
    }
    acc[(e >> 1) & 3] = add2(acc[(e >> 1) & 3], v);
  }
  const float2 s01 = add2(acc[0], acc[1]), s23 = add2(acc[2], acc[3]);
  const float2 s4 = add2(s01, s23);
  return s4.x + s4.y;
}

// ---- split scheduling: kernels over equal shares of the (pair, K/V tile) units ---
// With one CTA per pair of query tiles, a grid of P pairs fills ceil(P / SMs) waves
// and leaves SMs idle in the last one (P = 128 on 148 SMs: 14 % idle).  Here the
// (pair, K/V tile) units are cut into G contiguous ranges of equal length, one per SM,
// so a pair's slots may be spread over two or three CTAs ("segments").  The score-sum
// pass always runs this way (every slot sum is written by one CTA); the attention pass
// when the grid would leave a quarter of the SMs idle (its split pairs' (max, sum, O)
// pieces merged by combine_fwd_kernel).  The fused kernel's own split: kernel A runs
// phase A over each segment and stores the rows' partial (max, sum); kernel B combines
// a pair's partials into the final row LSE, runs phase B over its segments and writes
// y, or a partial O when the pair is split (the partials add up: P is already
// normalised); a reduction sums the partial O's.  The fused split requires an even
// number of query tiles per KV group (every pair has two tiles).
struct SplitParams {
  TcParams t;
  int G;            // CTAs (one per SM)
  int max_seg;      // segments per CTA at most
  long long U;      // units = pairs * n_kt
  float2 *part_ml;  // [G][max_seg][2 tiles][BM] (max, sum), base-2 units
  float *part_o;    // [G][max_seg][2 tiles][BM][D]
};

struct PairInfo {
  int bg, bhq_a, bhq_b, i0_a, i0_b, t_a, t_b;
};
__device__ __forceinline__ PairInfo pair_info(int pidx, const TcParams &p) {
  PairInfo r;
  r.bg = pidx / p.ctas_per_group;
  const int cpi = pidx - r.bg * p.ctas_per_group;
  const int b = r.bg / p.Hk, g = r.bg - b * p.Hk;
  const int qa = 2 * cpi, qb = qa + 1;
  const int hl_a = qa / p.tiles, hl_b = qb / p.tiles;
  r.t_a = qa - hl_a * p.tiles;
  r.t_b = qb - hl_b * p.tiles;
  r.bhq_a = b * p.Hq + g * p.q_g + hl_a;
  r.bhq_b = b * p.Hq + g * p.q_g + hl_b;
  r.i0_a = r.t_a * BM;
  r.i0_b = r.t_b * BM;
  return r;
}

// First unit of CTA c.
__device__ __forceinline__ long long unit0(int c, const SplitParams &sp) {
  return (sp.U * (long long)c) / sp.G;
}
// Segments of this CTA: pair p, tiles [kt0, kt1), and the segment's index in range
// order (its slot in the partial buffers).  A range that starts inside a pair
// processes that first piece last, so that every CTA sweeps its K/V tiles from tile 0
// upwards at about the same time as the others: the tiles a group's CTAs share are
// then read within a short window and stay in L2.
struct SegIter {
  long long u, u1;   // the rest of the range in natural order
  long long f0, f1;  // the rotated first piece (empty if none)
  long long ubase;   // first unit of the range
  int n_kt;
  __device__ __forceinline__ bool take(long long &a, long long b, int &p, int &kt0, int &kt1) {
    p = (int)(a / n_kt);
    kt0 = (int)(a - (long long)p * n_kt);
    kt1 = (int)min((long long)n_kt, kt0 + (b - a));
    a += kt1 - kt0;
    return true;
  }
  __device__ __forceinline__ bool next(int &p, int &kt0, int &kt1, int &slot) {
    if (u < u1) take(u, u1, p, kt0, kt1);
    else if (f0 < f1) take(f0, f1, p, kt0, kt1);
    else return false;
    slot = p - (int)(ubase / n_kt);
    return true;
  }
};
// The same segments with 32-bit unit indices (pass 1 holds it in every role).
struct SegIter32 {
  int u, u1, f0, f1, ubase, n_kt;
  __device__ __forceinline__ void take(int &a, int b, int &p, int &kt0, int &kt1) {
    p = a / n_kt;
    kt0 = a - p * n_kt;
    kt1 = min(n_kt, kt0 + (b - a));
    a += kt1 - kt0;
  }
  __device__ __forceinline__ bool next(int &p, int &kt0, int &kt1, int &slot) {
    if (u < u1) take(u, u1, p, kt0, kt1);
    else if (f0 < f1) take(f0, f1, p, kt0, kt1);
    else return false;
    slot = p - ubase / n_kt;
    return true;
  }
};
__device__ __forceinline__ SegIter32 seg_iter32(const SplitParams &sp) {
  SegIter32 it;
  it.n_kt = sp.t.n_kt;
  it.ubase = (int)unit0(blockIdx.x, sp);
  it.u1 = (int)unit0(blockIdx.x + 1, sp);
  const int kt0 = it.ubase % it.n_kt;
  const int first_end = min(it.u1, it.ubase + (it.n_kt - kt0));
  if (kt0 > 0 && first_end < it.u1) {
    it.f0 = it.ubase;
    it.f1 = first_end;
    it.u = first_end;
  } else {
    it.f0 = it.f1 = 0;
    it.u = it.ubase;
  }
  return it;
}
__device__ __forceinline__ SegIter seg_iter(const SplitParams &sp) {
  SegIter it;
  it.n_kt = sp.t.n_kt;
  it.ubase = unit0(blockIdx.x, sp);
  it.u1 = unit0(blockIdx.x + 1, sp);
  const long long kt0 = it.ubase % it.n_kt;
  const long long first_end = min(it.u1, it.ubase + (it.n_kt - kt0));
  if (kt0 > 0 && first_end < it.u1) {  // starts inside a pair and holds more
    it.f0 = it.ubase;
    it.f1 = first_end;
    it.u = first_end;
  } else {
    it.f0 = it.f1 = 0;
    it.u = it.ubase;
  }
  return it;
}
// CTAs whose ranges hold units of pair p: [c_first, c_last]; segment slot of p in c.
// Pass 2 over equal shares of the (pair, K tile) units: CTA c takes units
// [U c / G, U (c + 1) / G) in segments of one pair each, so that all
// SMs are busy whatever the number of pairs; each (row tile, slot) sum is written by
// exactly one CTA.  With G = pairs every CTA takes one whole pair.  Four softmax
// warpgroups: (tile, S^T buffer parity), so that each takes every other K tile of its
// query tile and four of them share each SM sub-partition's exponential unit.
__global__ void __launch_bounds__(kThreadsS, 1)
    scoresum_kernel(const __grid_constant__ CUtensorMap q_map,
                    const __grid_constant__ CUtensorMap k_map, const SplitParams sp) {
  const TcParams &p = sp.t;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicExch(p.status, H2OKV_ERR_CUDA);
    return;
  }
  float *nlse_s = reinterpret_cast<float *>(smem + S_OFF_NLSE);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + S_OFF_BAR);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + S_OFF_TMEM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = p.q_g * p.tiles;
  const uint64_t lim = p.timeout_ns;
  if (threadIdx.x == 0) {
    mbar_init(&bar[G_Q], 1);
    for (int i = 0; i < kStagesS; ++i) {
      mbar_init(&bar[G_KFULL0 + i], 1);
      mbar_init(&bar[G_KEMPTY0 + i], 1);  // the MMA's commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[G_SFULL0 + i], 1);
      mbar_init(&bar[G_SFREE0 + i], 8);  // both softmax warpgroups, with or without a tile
    }
    mbar_init(&bar[G_QFREE], 1);
    mbar_init(&bar[G_NL0], 8);  // both warpgroups of a tile
    mbar_init(&bar[G_NL0 + 1], 8);
    mbar_init(&bar[G_DRAIN], 1);
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
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_s;
  bool aborted = false;
  // this CTA's units, in natural order (every K tile of pass 2 fits in L2)
  const int n_kt = p.n_kt;
  const int u_first = (int)((sp.U * blockIdx.x) / sp.G), u_last = (int)((sp.U * (blockIdx.x + 1)) / sp.G);
  int pidx, kt0, kt1;
  auto next = [&](int &u) -> bool {
    if (u >= u_last) return false;
    pidx = u / n_kt;
    kt0 = u - pidx * n_kt;
    kt1 = min(n_kt, kt0 + (u_last - u));
    u += kt1 - kt0;
    return true;
  };

  if (warp < 4) {
    reg_dealloc<kCtrlRegsS>();
    if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      // S^T_t(i) = K Q_t^T of the CTA's i-th unit into columns 256 (i & 1) + 128 t
      if (lane == 0) {
        const uint32_t qa_addr = sbase + S_OFF_QA, qb_addr = sbase + S_OFF_QB;
        int i = 0, seg = 0, u = u_first;
        while (!aborted && next(u)) {
          const bool has_b = 2 * (pidx % p.ctas_per_group) + 1 < n_qt;
          if (!mbar_wait(&bar[G_Q], seg & 1, lim)) { fail(p, aborted); break; }
          tc_fence_after();
          for (int kt = kt0; kt < kt1 && !aborted; ++kt, ++i) {
            const int s = i % kStagesS, u = i & 1;
            if (!mbar_wait(&bar[G_KFULL0 + s], (i / kStagesS) & 1, lim)) { fail(p, aborted); break; }
            if (i >= 2 && !mbar_wait(&bar[G_SFREE0 + u], ((i >> 1) - 1) & 1, lim)) {
              fail(p, aborted);
              break;
            }
            tc_fence_after();
            const uint32_t k_addr = sbase + S_OFF_K + s * kTileBytes;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_bf16_ss(tmem + u * 256, kmajor_desc(k_addr, ks), kmajor_desc(qa_addr, ks),
                          IDESC_K_MAJOR, ks > 0);
            if (has_b) {
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                mma_bf16_ss(tmem + u * 256 + 128, kmajor_desc(k_addr, ks),
                            kmajor_desc(qb_addr, ks), IDESC_K_MAJOR, ks > 0);
            }
            mma_commit(&bar[G_SFULL0 + u]);
            mma_commit(&bar[G_KEMPTY0 + s]);
          }
          mma_commit(&bar[G_QFREE]);  // the segment's Q tiles no longer read
          ++seg;
        }
        mma_commit(&bar[G_DRAIN]);
        mbar_wait(&bar[G_DRAIN], 0, 4000000000ull);
      }
      __syncwarp();
    } else if (warp == 0) {
      // ---------------------------------------------- producer of Q (per segment) and K
      if (lane == 0) {
        int i = 0, seg = 0, u = u_first;
        while (!aborted && next(u)) {
          const PairInfo pi = pair_info(pidx, p);
          const bool has_b = 2 * (pidx % p.ctas_per_group) + 1 < n_qt;
          if (seg > 0 && !mbar_wait(&bar[G_QFREE], (seg - 1) & 1, lim)) { fail(p, aborted); break; }
          mbar_expect_tx(&bar[G_Q], has_b ? 2 * kTileBytes : kTileBytes);
          tma_load_3d(smem + S_OFF_QA, &q_map, &bar[G_Q], 0, pi.i0_a, pi.bhq_a);
          tma_load_3d(smem + S_OFF_QA + kHalfBytes, &q_map, &bar[G_Q], 64, pi.i0_a, pi.bhq_a);
          if (has_b) {
            tma_load_3d(smem + S_OFF_QB, &q_map, &bar[G_Q], 0, pi.i0_b, pi.bhq_b);
            tma_load_3d(smem + S_OFF_QB + kHalfBytes, &q_map, &bar[G_Q], 64, pi.i0_b, pi.bhq_b);
          }
          mbar_arrive(&bar[G_Q]);
          for (int kt = kt0; kt < kt1 && !aborted; ++kt, ++i) {
            const int s = i % kStagesS, n = i / kStagesS;
            if (n > 0 && !mbar_wait(&bar[G_KEMPTY0 + s], (n - 1) & 1, lim)) { fail(p, aborted); break; }
            uint8_t *kdst = smem + S_OFF_K + s * kTileBytes;
            mbar_expect_tx(&bar[G_KFULL0 + s], kTileBytes);
            tma_load_3d(kdst, &k_map, &bar[G_KFULL0 + s], 0, kt * BN, pi.bg);
            tma_load_3d(kdst + kHalfBytes, &k_map, &bar[G_KFULL0 + s], 64, kt * BN, pi.bg);
            if (kt + kPrefetch < kt1) {
              tma_prefetch_l2_3d(&k_map, 0, (kt + kPrefetch) * BN, pi.bg);
              tma_prefetch_l2_3d(&k_map, 64, (kt + kPrefetch) * BN, pi.bg);
            }
            mbar_arrive(&bar[G_KFULL0 + s]);
          }
          ++seg;
        }
        // drain: the last issued loads land before exit
        if (seg > 0) mbar_wait(&bar[G_Q], (seg - 1) & 1, 4000000000ull);
        for (int j = i - 1; j >= 0 && j >= i - kStagesS; --j)
          mbar_wait(&bar[G_KFULL0 + j % kStagesS], (j / kStagesS) & 1, 4000000000ull);
      }
      __syncwarp();
    }
  } else {
    reg_alloc<kSoftRegsS>();
    // ------------------------------------- column sums, one thread per slot of a tile
    const int wg = (warp - 4) >> 2;
    const int t = wg & 1, par = wg >> 1;  // query tile; parity of the units (S^T buffer) taken
    const int st = threadIdx.x & 127;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const float c2 = p.scale2;
    int i = 0, seg = 0, u = u_first;
    while (!aborted && next(u)) {
      const PairInfo pi = pair_info(pidx, p);
      const bool active = t == 0 || 2 * (pidx % p.ctas_per_group) + 1 < n_qt;
      const int i0 = t ? pi.i0_b : pi.i0_a, bhq = t ? pi.bhq_b : pi.bhq_a, tt = t ? pi.t_b : pi.t_a;
      // -lse2 of the segment's rows, double buffered by segment: a warpgroup writes
      // buffer seg & 1 only after all its threads have written (so finished reading)
      // the other one
      float *nl = nlse_s + ((seg & 1) * 2 + t) * BM;
      if (active) nl[st] = p.nlse[((size_t)bhq * p.tiles + tt) * BM + st];  // both warpgroups: same value
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[G_NL0 + t]);
      if (!warp_wait(&bar[G_NL0 + t], seg & 1, lim)) { fail(p, aborted); break; }
      ++seg;
      const int rmax = min(BM, p.S - i0);
      float *pw = p.part_w + ((size_t)bhq * p.tiles + tt) * p.N_C;
      // this warpgroup's K tiles: unit index i = i_seg + (kt - kt0) of parity par
      const int i_seg = i;
      i += kt1 - kt0;
      const int kt_first = kt0 + ((par - i_seg) & 1);
      // each slot's token position, read one of our K tiles ahead (empty / outside: far)
      const int32_t *tpg = p.token_pos + (size_t)pi.bg * p.N_C;
      int32_t tp_next = kt_first < kt1 && kt_first * BN + st < p.N_C ? tpg[kt_first * BN + st] : kEmptyPos;
      for (int kt = kt_first; kt < kt1; kt += 2) {
        const int iu = i_seg + (kt - kt0);
        const int u = iu & 1;
        const int j = kt * BN + st;
        const int32_t tp = tp_next;
        if (kt + 2 < kt1) tp_next = j + 2 * BN < p.N_C ? tpg[j + 2 * BN] : kEmptyPos;
        if (!warp_wait(&bar[G_SFULL0 + u], (iu >> 1) & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        if (active) {
          // visible rows r of this tile: tp - P <= i0 + r, r < rmax.  A slot that no row
          // of the tile sees (a later token of the chunk, an empty slot) sums to 0 and
          // needs no masking; only slots first seen inside the tile do.
          const int64_t rel = (int64_t)tp - (int64_t)p.P - (int64_t)i0;
          const int rmin = rel <= 0 ? 0 : (rel >= BM ? BM : (int)rel);
          const bool none = rmin >= rmax;
          const bool full = __all_sync(0xffffffffu, (rmin == 0 || none) && rmax == BM);
          // the tile's 128 rows in two halves of 64 (fewer live registers)
          const uint32_t ta = tmem + lane_base + u * 256 + t * 128;
          float cs = 0.f;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t r[BM / 2];
            tmem_ld32(ta + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(r));
            tmem_ld32(ta + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
            tmem_wait_ld();
            if (h == 1) {  // the S^T buffer is free once read
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bar[G_SFREE0 + u]);
            }
            cs += full ? slot_colsum<false>(r, nl + 64 * h, c2, 0, BM / 2)
                       : slot_colsum<true>(r, nl + 64 * h, c2, rmin - 64 * h, rmax - 64 * h);
          }
          if (j < p.N_C) pw[j] = none ? 0.f : cs;
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[G_SFREE0 + u]);
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

__device__ __forceinline__ int cta_of_unit(long long x, const SplitParams &sp) {
  // largest c with floor(U c / G) <= x
  return (int)(((x + 1) * sp.G + sp.U - 1) / sp.U) - 1;
}
__device__ __forceinline__ int seg_slot(int p, int c, const SplitParams &sp) {
  return p - (int)(unit0(c, sp) / sp.t.n_kt);
}

// Pass 1 over equal shares of the (pair, K/V tile) units, one CTA per SM: CTA c takes
// units [U c / G, U (c + 1) / G) in segments of one pair each (SegIter order).  A
// segment that covers a whole pair writes y and -lse2; the pieces of a pair split over
// CTAs write their rows' (max, sum) and unnormalised O, which combine_fwd_kernel
// merges.  With G = pairs every CTA takes one whole pair.
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap q_map,
                    const __grid_constant__ CUtensorMap k_map,
                    const __grid_constant__ CUtensorMap v_map, const SplitParams sp) {
  const TcParams &p = sp.t;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicExch(p.status, H2OKV_ERR_CUDA);
    return;
  }
  float *rel_s = reinterpret_cast<float *>(smem + F_OFF_REL);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + F_OFF_BAR);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + F_OFF_TMEM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = p.q_g * p.tiles;
  const int n_kt = p.n_kt;
  const uint64_t lim = p.timeout_ns;
  int4 *segs = reinterpret_cast<int4 *>(smem + F_OFF_SEG);
  if (threadIdx.x == 0) {
    SegIter32 it = seg_iter32(sp);
    int n = 0, pp, a0, a1, sl;
    while (n < kMaxSegF && it.next(pp, a0, a1, sl)) segs[1 + n++] = make_int4(pp, a0, a1, sl);
    segs[0].x = n;
    mbar_init(&bar[F_Q], 1);
    for (int i = 0; i < kStagesF; ++i) {
      mbar_init(&bar[F_KFULL0 + i], 1);
      mbar_init(&bar[F_KEMPTY0 + i], 1 + 8);  // MMA commit + all softmax warps (positions)
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[F_VFULL0 + i], 1);
      mbar_init(&bar[F_VEMPTY0 + i], 1);
      mbar_init(&bar[F_SFULL0 + i], 1);
      mbar_init(&bar[F_PFULL0 + i], 4);
    }
    mbar_init(&bar[F_OFULL], 1);
    mbar_init(&bar[F_OFREE], 8);
    mbar_init(&bar[F_QFREE], 1);
    mbar_init(&bar[F_DRAIN], 1);
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
  const int nseg = segs[0].x;
  int pidx, kt0, kt1, slot;
  auto segment = [&](int sg) {
    const int4 e = segs[1 + sg];
    pidx = e.x;
    kt0 = e.y;
    kt1 = e.z;
    slot = e.w;
  };

  if (warp < 4) {
    reg_dealloc<kCtrlRegsF>();
    if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      // TMEM columns: S / P of tile a at 0, of tile b at 128; O of tile a at 256, b at 384.
      if (lane == 0) {
        const uint32_t qa_addr = sbase + F_OFF_QA, qb_addr = sbase + F_OFF_QB;
        int ibase = 0, nb_base = 0;  // units before this segment (all / tile b)
        for (int seg = 0; seg < nseg && !aborted; ++seg) {
          segment(seg);
          const bool has_b = 2 * (pidx % p.ctas_per_group) + 1 < n_qt;
          const int len = kt1 - kt0;
          // S_t of the segment's first tile.  Every later S_t(kt+1) is issued after
          // P_t(kt) V: the tensor core runs one thread's MMAs in order, so P (which
          // overlays S) is read before it is overwritten.
          if (!mbar_wait(&bar[F_Q], seg & 1, lim) ||
              !mbar_wait(&bar[F_KFULL0 + ibase % kStagesF], (ibase / kStagesF) & 1, lim)) {
            fail(p, aborted);
            break;
          }
          tc_fence_after();
          {
            const uint32_t k_addr = sbase + F_OFF_K + (ibase % kStagesF) * kTileBytes;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (t == 1 && !has_b) break;
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                mma_bf16_ss(tmem + t * 128, kmajor_desc(t ? qb_addr : qa_addr, ks),
                            kmajor_desc(k_addr, ks), IDESC_K_MAJOR, ks > 0);
              mma_commit(&bar[F_SFULL0 + t]);
            }
            mma_commit(&bar[F_KEMPTY0 + ibase % kStagesF]);  // first K no longer read
          }
          // O of the previous segment read out before the first P V overwrites it
          if (seg > 0 && !mbar_wait(&bar[F_OFREE], (seg - 1) & 1, lim)) { fail(p, aborted); break; }
          // Per query tile and K/V tile: O_t (+)= P_t V (A from TMEM, 16 slots = 8
          // columns per k-step) and S_t of the next tile.  The tiles are served in the
          // order their P arrives: the barriers are polled, never waited on, so a tile
          // that runs ahead (as far as the K / V rings allow) never holds up the other.
          // The K and V stages are released by the second tile's commit.
          int np0 = 0, np1 = has_b ? 0 : len;  // next P V of tile a / b, within the segment
          uint64_t t_last = globaltimer();
          while (!aborted && (np0 < len || np1 < len)) {
            bool progressed = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int k = t ? np1 : np0;
              if (k >= len) continue;
              const int i = ibase + k;                        // unit index in the CTA
              const int n = (t ? nb_base : ibase) + k;        // this tile's P count
              const bool more = k + 1 < len;
              const int v = i & 1, s1 = (i + 1) % kStagesF;
              if (!mbar_test(&bar[F_PFULL0 + t], n & 1) ||
                  !mbar_test(&bar[F_VFULL0 + v], (i >> 1) & 1) ||
                  (more && !mbar_test(&bar[F_KFULL0 + s1], ((i + 1) / kStagesF) & 1)))
                continue;
              tc_fence_after();
              const uint32_t v_addr = sbase + F_OFF_V + v * kTileBytes;
#pragma unroll
              for (int ks = 0; ks < BN / 16; ++ks)
                mma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + ks * 8, mnmajor_desc(v_addr, ks),
                            IDESC_TS_PV, (k > 0 || ks > 0) ? 1u : 0u);
              // the other tile has issued its P V and next S already
              const bool second = (t ? np0 : np1) > k;
              if (second) mma_commit(&bar[F_VEMPTY0 + v]);  // V no longer read
              if (more) {
                const uint32_t k_addr = sbase + F_OFF_K + s1 * kTileBytes;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                  mma_bf16_ss(tmem + t * 128, kmajor_desc(t ? qb_addr : qa_addr, ks),
                              kmajor_desc(k_addr, ks), IDESC_K_MAJOR, ks > 0);
                mma_commit(&bar[F_SFULL0 + t]);
                if (second) mma_commit(&bar[F_KEMPTY0 + s1]);  // K no longer read
              }
              if (t) np1 = k + 1; else np0 = k + 1;
              progressed = true;
            }
            const uint64_t now = globaltimer();
            if (progressed) t_last = now;
            else if (now - t_last > lim) fail(p, aborted);
          }
          mma_commit(&bar[F_OFULL]);
          mma_commit(&bar[F_QFREE]);  // the segment's Q tiles no longer read
          ibase += len;
          if (has_b) nb_base += len;
        }
        mma_commit(&bar[F_DRAIN]);
        mbar_wait(&bar[F_DRAIN], 0, 4000000000ull);
      }
      __syncwarp();
    } else if (warp == 0) {
      // ------------------------- producer of Q (per segment), K and slot positions
      int i = 0, seg = 0;
      for (; seg < nseg && !aborted; ++seg) {
        segment(seg);
        const PairInfo pi = pair_info(pidx, p);
        const bool has_b = 2 * (pidx % p.ctas_per_group) + 1 < n_qt;
        if (seg > 0 && !warp_wait(&bar[F_QFREE], (seg - 1) & 1, lim)) { fail(p, aborted); break; }
        if (lane == 0) {
          mbar_expect_tx(&bar[F_Q], has_b ? 2 * kTileBytes : kTileBytes);
          tma_load_3d(smem + F_OFF_QA, &q_map, &bar[F_Q], 0, pi.i0_a, pi.bhq_a);
          tma_load_3d(smem + F_OFF_QA + kHalfBytes, &q_map, &bar[F_Q], 64, pi.i0_a, pi.bhq_a);
          if (has_b) {
            tma_load_3d(smem + F_OFF_QB, &q_map, &bar[F_Q], 0, pi.i0_b, pi.bhq_b);
            tma_load_3d(smem + F_OFF_QB + kHalfBytes, &q_map, &bar[F_Q], 64, pi.i0_b, pi.bhq_b);
          }
          mbar_arrive(&bar[F_Q]);
        }
        const int32_t *tpg = p.token_pos + (size_t)pi.bg * p.N_C;
        const float thr = (float)(has_b ? min(pi.i0_a, pi.i0_b) : pi.i0_a);
        for (int kt = kt0; kt < kt1 && !aborted; ++kt, ++i) {
          const int s = i % kStagesF, n = i / kStagesF;
          if (n > 0 && !warp_wait(&bar[F_KEMPTY0 + s], (n - 1) & 1, lim)) { fail(p, aborted); break; }
          uint8_t *kdst = smem + F_OFF_K + s * kTileBytes;
          if (lane == 0) {
            mbar_expect_tx(&bar[F_KFULL0 + s], kTileBytes);
            tma_load_3d(kdst, &k_map, &bar[F_KFULL0 + s], 0, kt * BN, pi.bg);
            tma_load_3d(kdst + kHalfBytes, &k_map, &bar[F_KFULL0 + s], 64, kt * BN, pi.bg);
            if (kt + kPrefetch < kt1) {
              tma_prefetch_l2_3d(&k_map, 0, (kt + kPrefetch) * BN, pi.bg);
              tma_prefetch_l2_3d(&k_map, 64, (kt + kPrefetch) * BN, pi.bg);
            }
          }
          tile_positions(rel_s + s * BN, tpg, kt, p.N_C, p.P, lane);
          __syncwarp();
          {
            // slots invisible to the first row of a tile, compacted in slot order
            int32_t *cand = reinterpret_cast<int32_t *>(smem + F_OFF_CAND) + s * kCandWords;
            int total = 0;
#pragma unroll 1
            for (int q = 0; q < 4; ++q)
              total += __popc(__ballot_sync(0xffffffffu, rel_s[s * BN + lane + 32 * q] > thr));
            if (total <= kMaxCand) {
              int off = 0;
#pragma unroll 1
              for (int q = 0; q < 4; ++q) {
                const float rq = rel_s[s * BN + lane + 32 * q];
                const uint32_t bq = __ballot_sync(0xffffffffu, rq > thr);
                if ((bq >> lane) & 1u) {
                  const int idx = off + __popc(bq & ((1u << lane) - 1u));
                  cand[2 + 2 * idx] = lane + 32 * q;
                  cand[3 + 2 * idx] = __float_as_int(rq);
                }
                off += __popc(bq);
              }
            }
            if (lane == 0) cand[0] = total <= kMaxCand ? total : -1;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[F_KFULL0 + s]);
        }
      }
      // drain: the last issued loads land before exit
      if (lane == 0) {
        if (seg > 0) mbar_wait(&bar[F_Q], (seg - 1) & 1, 4000000000ull);
        for (int j = i - 1; j >= 0 && j >= i - kStagesF; --j)
          mbar_wait(&bar[F_KFULL0 + j % kStagesF], (j / kStagesF) & 1, 4000000000ull);
      }
    } else if (warp == 2) {
      // ------------------------------------------------------------------ producer of V
      if (lane == 0) {
        int i = 0;
        for (int sg = 0; sg < nseg && !aborted; ++sg) {
          segment(sg);
          const int bg = pidx / p.ctas_per_group;
          for (int kt = kt0; kt < kt1 && !aborted; ++kt, ++i) {
            const int v = i & 1, n = i >> 1;
            if (n > 0 && !mbar_wait(&bar[F_VEMPTY0 + v], (n - 1) & 1, lim)) { fail(p, aborted); break; }
            uint8_t *vdst = smem + F_OFF_V + v * kTileBytes;
            mbar_expect_tx(&bar[F_VFULL0 + v], kTileBytes);
            tma_load_3d(vdst, &v_map, &bar[F_VFULL0 + v], 0, kt * BN, bg);
            tma_load_3d(vdst + kHalfBytes, &v_map, &bar[F_VFULL0 + v], 64, kt * BN, bg);
            mbar_arrive(&bar[F_VFULL0 + v]);
            if (kt + kPrefetch < kt1) {
              tma_prefetch_l2_3d(&v_map, 0, (kt + kPrefetch) * BN, bg);
              tma_prefetch_l2_3d(&v_map, 64, (kt + kPrefetch) * BN, bg);
            }
          }
        }
        for (int j = i - 1; j >= 0 && j >= i - 2; --j)
          mbar_wait(&bar[F_VFULL0 + (j & 1)], (j >> 1) & 1, 4000000000ull);
      }
      __syncwarp();
    }
  } else {
    reg_alloc<kSoftRegsF>();
    const int t = (warp - 4) >> 2;  // 0: tile a, 1: tile b
    // ------------------------------------- online softmax, one thread per query row
    const int st = threadIdx.x - 128 * (1 + t);
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t s_col = tmem + lane_base + t * 128, o_col = tmem + lane_base + 256 + t * 128;
    const float c2 = p.scale2;
    const float mbias = kMaskBias / c2;
    int i = 0, nt = 0;  // units of the CTA, units of this tile
    for (int seg = 0; seg < nseg && !aborted; ++seg) {
      segment(seg);
      const PairInfo pi = pair_info(pidx, p);
      const bool active = t == 0 || 2 * (pidx % p.ctas_per_group) + 1 < n_qt;
      if (!active) {
        // no tile b in this pair: keep the position ring's count
        for (int kt = kt0; kt < kt1; ++kt, ++i) {
          const int s = i % kStagesF;
          if (!warp_wait(&bar[F_KFULL0 + s], (i / kStagesF) & 1, lim)) { fail(p, aborted); break; }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[F_KEMPTY0 + s]);
        }
        if (!aborted && !warp_wait(&bar[F_OFULL], seg & 1, lim)) fail(p, aborted);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[F_OFREE]);
        continue;
      }
      const int i0 = t ? pi.i0_b : pi.i0_a, bhq = t ? pi.bhq_b : pi.bhq_a, tt = t ? pi.t_b : pi.t_a;
      float m = -INFINITY, l = 0.f;  // reference maximum (base 2) and sum against it
      uint32_t x[BN];
      for (int kt = kt0; kt < kt1 && !aborted; ++kt, ++i, ++nt) {
        const int s = i % kStagesF;
        if (!warp_wait(&bar[F_SFULL0 + t], nt & 1, lim)) { fail(p, aborted); break; }
        if (!warp_wait(&bar[F_KFULL0 + s], (i / kStagesF) & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        const float *rel = rel_s + s * BN;
        const int32_t *cand = reinterpret_cast<const int32_t *>(smem + F_OFF_CAND) + s * kCandWords;
        const int nc = cand[0];
        if (nc > 0) {
          // few slots to mask: lower them in TMEM before the row is read (a masked
          // logit drops by 2^30 in base-2 units, as in row_mask)
          const float ri = (float)(i0 + st);
#pragma unroll 1
          for (int q0 = 0; q0 < nc; q0 += 4) {
            uint32_t cv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (q0 + q < nc) cv[q] = tmem_ld1(s_col + cand[2 + 2 * (q0 + q)]);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (q0 + q < nc) {
                const float nm = fma_sat(__int_as_float(cand[3 + 2 * (q0 + q)]), 1.f, -ri);
                tmem_st1(s_col + cand[2 + 2 * (q0 + q)],
                         __float_as_uint(fmaf(nm, -mbias, __uint_as_float(cv[q]))));
              }
          }
          tmem_wait_st();
        }
        const bool masked = nc < 0;  // too many: mask the whole row after reading it
        tmem_ld32(s_col, *reinterpret_cast<uint32_t(*)[32]>(x));
        tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
        tmem_ld32(s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(x + 64));
        tmem_ld32(s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(x + 96));
        tmem_wait_ld();
        if (masked) row_mask<BN>(x, rel, (float)(i0 + st), mbias);
        // Probabilities against the reference maximum m, computed alongside the row
        // maximum.  m follows the row maximum lazily (p <= 2^8 in between); when the
        // maximum exceeds it by more than that (the first tile; rarely later) m moves,
        // O and l are rescaled and the tile is done again from S, still in TMEM.
        uint32_t pk[BN / 2];
        const float mx = row_max<BN>(x) * c2;
        float ps = row_probs(x, c2, m, pk);
        const bool need = mx > m + kLazyMax;
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = need ? mx : m;
          const float f = ex2(m - m_new);  // 1 if unchanged, 0 from -inf
          l *= f;
          if (kt > kt0) {
            // O holds the sums of P V up to the previous tile: every MMA before S(kt)
            // is complete, none after it is issued until this warp's P is written
#pragma unroll 1
            for (int cq = 0; cq < 4; ++cq) {
              uint32_t o[32];
              tmem_ld32(o_col + cq * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
              tmem_st32(o_col + cq * 32, o);
            }
          }
          m = m_new;
          tmem_ld32(s_col, *reinterpret_cast<uint32_t(*)[32]>(x));
          tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
          tmem_ld32(s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(x + 64));
          tmem_ld32(s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(x + 96));
          tmem_wait_ld();
          if (masked) row_mask<BN>(x, rel, (float)(i0 + st), mbias);
          ps = row_probs(x, c2, m, pk);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[F_KEMPTY0 + s]);  // positions no longer read
        // P over S (bf16 pairs), the A operand of O += P V
        tmem_st32(s_col, *reinterpret_cast<uint32_t(*)[32]>(pk));
        tmem_st32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
        l += ps;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[F_PFULL0 + t]);
      }
      if (aborted) break;
      // the segment's rows: y, -lse2 and lse for a whole pair, else the piece's
      // (max, sum) and O for combine_fwd_kernel
      const bool whole = kt0 == 0 && kt1 == n_kt;
      const bool row_ok = i0 + st < p.S;
      if (!warp_wait(&bar[F_OFULL], seg & 1, lim)) { fail(p, aborted); break; }
      tc_fence_after();
      if (whole) {
        const bool seen = l > 0.f && m > -0.5f * kMaskBias;
        const float lse2 = seen ? m + lg2(l) : -INFINITY;
        p.nlse[((size_t)bhq * p.tiles + tt) * BM + st] = seen ? -lse2 : -kMaskBias;
        if (p.lse_out && row_ok) p.lse_out[(size_t)bhq * p.S + i0 + st] = lse2 * 0.69314718055994531f;
        const float inv = seen ? 1.f / l : 0.f;
        __nv_bfloat16 *yrow = p.y + ((size_t)bhq * p.S + i0 + st) * D;
        uint32_t r[32];
#pragma unroll
        for (int cq = 0; cq < 4; ++cq) {
          tmem_ld32(o_col + cq * 32, r);
          tmem_wait_ld();
          if (row_ok) {
            uint32_t o[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              o[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv, __uint_as_float(r[2 * e + 1]) * inv);
            uint4 *dst = reinterpret_cast<uint4 *>(yrow + cq * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
          }
        }
      } else {
        const size_t prow = (((size_t)blockIdx.x * sp.max_seg + slot) * 2 + t) * BM + st;
        sp.part_ml[prow] = make_float2(m, l);
        float4 *dst = reinterpret_cast<float4 *>(sp.part_o + prow * D);
        uint32_t r[32];
#pragma unroll
        for (int cq = 0; cq < 4; ++cq) {
          tmem_ld32(o_col + cq * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[cq * 8 + e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                          __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[F_OFREE]);  // O read out
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// The pieces of every pair that pass 1 split over CTAs: per row, with the pieces'
// maxima m_i and sums l_i against them, m = max m_i, l = sum l_i 2^(m_i - m),
// O = sum O_i 2^(m_i - m); y = O / l, lse2 = m + log2 l.  Grid (pairs, 32): a CTA
// looks the pair's pieces up once; each thread takes one row and 4 columns.
constexpr int kMaxPieces = 8;
constexpr int kMinSplitTiles = 32;  // pass 1 is split over CTAs only for scans this long
__global__ void __launch_bounds__(256)
    combine_fwd_kernel(const SplitParams sp) {
  const TcParams &p = sp.t;
  const int pidx = blockIdx.x;
  __shared__ int piece_row[kMaxPieces];  // first partial row of each piece
  __shared__ int n_pieces;
  if (threadIdx.x == 0) {
    const int c_first = cta_of_unit((long long)pidx * p.n_kt, sp);
    const int c_last = cta_of_unit((long long)(pidx + 1) * p.n_kt - 1, sp);
    int n = 0;
    for (int c = c_first; c <= c_last && n < kMaxPieces; ++c, ++n)
      piece_row[n] = ((c * sp.max_seg + seg_slot(pidx, c, sp)) * 2) * BM;
    n_pieces = c_last > c_first ? n : 0;  // a pair of one piece was written by its CTA
  }
  __syncthreads();
  const int np = n_pieces;
  if (np == 0) return;
  const bool has_b = 2 * (pidx % p.ctas_per_group) + 1 < p.q_g * p.tiles;
  const PairInfo pi = pair_info(pidx, p);
  {
    const int e = blockIdx.y * blockDim.x + threadIdx.x;  // < 2 * BM * (D / 4)
    const int t = e / (BM * (D / 4));
    const int row = (e / (D / 4)) % BM, c4 = e % (D / 4);
    if (t == 1 && !has_b) return;
    const int i0 = t ? pi.i0_b : pi.i0_a, bhq = t ? pi.bhq_b : pi.bhq_a, tt = t ? pi.t_b : pi.t_a;
    float m = -INFINITY;
    for (int q = 0; q < np; ++q) m = fmaxf(m, sp.part_ml[piece_row[q] + t * BM + row].x);
    float l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < np; ++q) {
      const size_t prow = (size_t)piece_row[q] + t * BM + row;
      const float2 ml = sp.part_ml[prow];
      const float w = m == -INFINITY ? 0.f : ex2(ml.x - m);
      l += ml.y * w;
      const float4 v = __ldcs(reinterpret_cast<const float4 *>(sp.part_o + prow * D) + c4);
      acc.x += v.x * w;
      acc.y += v.y * w;
      acc.z += v.z * w;
      acc.w += v.w * w;
    }
    const bool seen = l > 0.f && m > -0.5f * kMaskBias;
    const float lse2 = seen ? m + lg2(l) : -INFINITY;
    if (c4 == 0) {
      p.nlse[((size_t)bhq * p.tiles + tt) * BM + row] = seen ? -lse2 : -kMaskBias;
      if (p.lse_out && i0 + row < p.S)
        p.lse_out[(size_t)bhq * p.S + i0 + row] = lse2 * 0.69314718055994531f;
    }
    if (i0 + row >= p.S) return;
    const float inv = seen ? 1.f / l : 0.f;
    __nv_bfloat162 *dst =
        reinterpret_cast<__nv_bfloat162 *>(p.y + ((size_t)bhq * p.S + i0 + row) * D + c4 * 4);
    dst[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    dst[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  }
}

enum {
  SA_Q = 0, SA_QFREE, SA_SFULL0, SA_SFULL1, SA_SFREE0, SA_SFREE1, SA_DRAIN,
  SA_AFULL0, SA_AEMPTY0 = SA_AFULL0 + kStagesA, SA_END = SA_AEMPTY0 + kStagesA
};
static_assert(SA_END <= NBAR, "split A barriers");

__global__ void __launch_bounds__(kThreads, 1)
    attn_split_a_kernel(const __grid_constant__ CUtensorMap q_map,
                        const __grid_constant__ CUtensorMap k_map, const SplitParams sp) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const TcParams &p = sp.t;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicExch(p.status, H2OKV_ERR_CUDA);
    return;
  }
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + OFF_TMEM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.timeout_ns;
  if (threadIdx.x == 0) {
    mbar_init(&bar[SA_Q], 1);
    mbar_init(&bar[SA_QFREE], 1);
    mbar_init(&bar[SA_DRAIN], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[SA_SFULL0 + i], 1);
      mbar_init(&bar[SA_SFREE0 + i], 8);
    }
    for (int i = 0; i < kStagesA; ++i) {
      mbar_init(&bar[SA_AFULL0 + i], 1);
      mbar_init(&bar[SA_AEMPTY0 + i], 1 + 8);
    }
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
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_s;
  bool aborted = false;

  if (warp < 4) {
    reg_dealloc<kCtrlRegs>();
    if (warp == 0) {
      // ---------------------------------------- Q per segment, K tiles, token positions
      SegIter si = seg_iter(sp);
      int pidx, kt0, kt1, slot, sidx = 0, it = 0;
      while (!aborted && si.next(pidx, kt0, kt1, slot)) {
        const PairInfo pi = pair_info(pidx, p);
        if (sidx > 0 && !warp_wait(&bar[SA_QFREE], (sidx - 1) & 1, lim)) { fail(p, aborted); break; }
        if (lane == 0) {
          mbar_expect_tx(&bar[SA_Q], 2 * kTileBytes);
          tma_load_3d(smem + OFF_QA, &q_map, &bar[SA_Q], 0, pi.i0_a, pi.bhq_a);
          tma_load_3d(smem + OFF_QA + kHalfBytes, &q_map, &bar[SA_Q], 64, pi.i0_a, pi.bhq_a);
          tma_load_3d(smem + OFF_QB, &q_map, &bar[SA_Q], 0, pi.i0_b, pi.bhq_b);
          tma_load_3d(smem + OFF_QB + kHalfBytes, &q_map, &bar[SA_Q], 64, pi.i0_b, pi.bhq_b);
          mbar_arrive(&bar[SA_Q]);
        }
        const int32_t *tpg = p.token_pos + (size_t)pi.bg * p.N_C;
        for (int kt = kt0; kt < kt1; ++kt, ++it) {
          const int stage = it % kStagesA, n = it / kStagesA;
          if (n > 0 && !warp_wait(&bar[SA_AEMPTY0 + stage], (n - 1) & 1, lim)) { fail(p, aborted); break; }
          uint64_t *full = &bar[SA_AFULL0 + stage];
          uint8_t *kdst = smem + slot_a(stage);
          if (lane == 0) {
            mbar_expect_tx(full, kTileBytes);
            tma_load_3d(kdst, &k_map, full, 0, kt * BN, pi.bg);
            tma_load_3d(kdst + kHalfBytes, &k_map, full, 64, kt * BN, pi.bg);
            if (kt + kPrefetch < kt1) {
              tma_prefetch_l2_3d(&k_map, 0, (kt + kPrefetch) * BN, pi.bg);
              tma_prefetch_l2_3d(&k_map, 64, (kt + kPrefetch) * BN, pi.bg);
            }
          }
          const int nv = min(BN, p.N_C - kt * BN);
          float *rel = reinterpret_cast<float *>(smem + OFF_REL_A) + stage * BN;
#pragma unroll
          for (int e = lane; e < BN; e += 32) {
            const int64_t t = e < nv ? (int64_t)tpg[kt * BN + e] : (int64_t)kEmptyPos;
            const int64_t r = t - (int64_t)p.P;
            rel[e] = (float)(r < -1 ? -1 : (r > kRelFar ? kRelFar : r));
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(full);
        }
        ++sidx;
      }
      // drain: the copies in flight land before exit
      if (lane == 0 && sidx > 0) {
        mbar_wait(&bar[SA_Q], (sidx - 1) & 1, 4000000000ull);
        for (int k = it - 1; k >= 0 && k >= it - kStagesA; --k)
          mbar_wait(&bar[SA_AFULL0 + k % kStagesA], (k / kStagesA) & 1, 4000000000ull);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t qa_addr = sbase + OFF_QA, qb_addr = sbase + OFF_QB;
        SegIter si = seg_iter(sp);
        int pidx, kt0, kt1, slot, sidx = 0, it = 0;
        while (!aborted && si.next(pidx, kt0, kt1, slot)) {
          if (!mbar_wait(&bar[SA_Q], sidx & 1, lim)) { fail(p, aborted); break; }
          tc_fence_after();
          for (int kt = kt0; kt < kt1; ++kt, ++it) {
            const int a = it % kStagesA, u = it & 1;
            if (!mbar_wait(&bar[SA_AFULL0 + a], (it / kStagesA) & 1, lim)) { fail(p, aborted); break; }
            if (it >= 2 && !mbar_wait(&bar[SA_SFREE0 + u], ((it >> 1) - 1) & 1, lim)) {
              fail(p, aborted);
              break;
            }
            tc_fence_after();
            const uint32_t k_addr = sbase + slot_a(a);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_bf16_ss(tmem + u * 256, kmajor_desc(qa_addr, ks), kmajor_desc(k_addr, ks),
                          IDESC_K_MAJOR, ks > 0);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_bf16_ss(tmem + u * 256 + 128, kmajor_desc(qb_addr, ks), kmajor_desc(k_addr, ks),
                          IDESC_K_MAJOR, ks > 0);
            mma_commit(&bar[SA_SFULL0 + u]);
            mma_commit(&bar[SA_AEMPTY0 + a]);
          }
          mma_commit(&bar[SA_QFREE]);  // this segment's Q tiles are no longer read
          ++sidx;
        }
        mma_commit(&bar[SA_DRAIN]);
        mbar_wait(&bar[SA_DRAIN], 0, 4000000000ull);
      }
      __syncwarp();
    }
  } else {
    reg_alloc<kSoftRegs>();
    // ---------------------------- online (max, sum) per row, one warpgroup per query tile
    const int wg = (warp - 4) >> 2;
    const int st = threadIdx.x - 128 * (1 + wg);
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const float c2 = p.scale2;
    const float mbias = kMaskBias / c2;
    SegIter si = seg_iter(sp);
    int pidx, kt0, kt1, slot, sidx = 0, it = 0;
    uint32_t x[BN];
    while (!aborted && si.next(pidx, kt0, kt1, slot)) {
      const PairInfo pi = pair_info(pidx, p);
      const int i0 = wg ? pi.i0_b : pi.i0_a;
      float m = -INFINITY, l = 0.f;
      for (int kt = kt0; kt < kt1 && !aborted; ++kt, ++it) {
        const int u = it & 1, a = it % kStagesA;
        if (!warp_wait(&bar[SA_SFULL0 + u], (it >> 1) & 1, lim)) { fail(p, aborted); break; }
        if (!warp_wait(&bar[SA_AFULL0 + a], (it / kStagesA) & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        const float *rela = reinterpret_cast<const float *>(smem + OFF_REL_A) + a * BN;
        const float rv = fmax3(fmaxf(rela[lane], rela[lane + 32]), rela[lane + 64], rela[lane + 96]);
        const bool masked = __any_sync(0xffffffffu, rv > (float)i0);
        const uint32_t sa = tmem + lane_base + u * 256 + wg * 128;
        tmem_ld32(sa, *reinterpret_cast<uint32_t(*)[32]>(x));
        tmem_ld32(sa + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
        tmem_ld32(sa + 64, *reinterpret_cast<uint32_t(*)[32]>(x + 64));
        tmem_ld32(sa + 96, *reinterpret_cast<uint32_t(*)[32]>(x + 96));
        tmem_wait_ld();
        if (masked) row_mask<BN>(x, rela, (float)(i0 + st), mbias);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar[SA_SFREE0 + u]);
          mbar_arrive(&bar[SA_AEMPTY0 + a]);
        }
        row_update<BN>(x, c2, m, l);
      }
      if (aborted) break;
      sp.part_ml[((size_t)blockIdx.x * sp.max_seg + slot) * (2 * BM) + wg * BM + st] = make_float2(m, l);
      ++sidx;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

enum {
  SB_Q = 0, SB_QFREE, SB_KFULL0, SB_KFULL1, SB_KEMPTY0, SB_KEMPTY1, SB_VFULL0, SB_VFULL1,
  SB_VEMPTY0, SB_VEMPTY1, SB_TFULLA, SB_TFULLB, SB_TFREEA, SB_TFREEB, SB_PFULLA, SB_PFULLB,
  SB_PFREEA, SB_PFREEB, SB_OFULL, SB_OFREE, SB_DRAIN, SB_END
};
static_assert(SB_END <= NBAR, "split B barriers");

__global__ void __launch_bounds__(kThreads, 1)
    attn_split_b_kernel(const __grid_constant__ CUtensorMap q_map,
                        const __grid_constant__ CUtensorMap k_map,
                        const __grid_constant__ CUtensorMap v_map, const SplitParams sp) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const TcParams &p = sp.t;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicExch(p.status, H2OKV_ERR_CUDA);
    return;
  }
  int32_t *tp_s = reinterpret_cast<int32_t *>(smem + OFF_TP);
  float *lse_s = reinterpret_cast<float *>(smem + OFF_LSE);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(smem + OFF_TMEM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.timeout_ns;
  if (threadIdx.x == 0) {
    mbar_init(&bar[SB_Q], 1);
    mbar_init(&bar[SB_QFREE], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[SB_KFULL0 + i], 1);
      mbar_init(&bar[SB_KEMPTY0 + i], 1 + 8);  // MMA commit + softmax warps (token positions)
      mbar_init(&bar[SB_VFULL0 + i], 1);
      mbar_init(&bar[SB_VEMPTY0 + i], 1);
    }
    mbar_init(&bar[SB_TFULLA], 1);
    mbar_init(&bar[SB_TFULLB], 1);
    mbar_init(&bar[SB_TFREEA], 4);
    mbar_init(&bar[SB_TFREEB], 4);
    mbar_init(&bar[SB_PFULLA], 4);
    mbar_init(&bar[SB_PFULLB], 4);
    mbar_init(&bar[SB_PFREEA], 1);
    mbar_init(&bar[SB_PFREEB], 1);
    mbar_init(&bar[SB_OFULL], 1);
    mbar_init(&bar[SB_OFREE], 8);
    mbar_init(&bar[SB_DRAIN], 1);
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

  if (warp < 4) {
    reg_dealloc<kCtrlRegs>();
    if (warp == 0) {
      // ---------------------------------------- Q per segment, K tiles, token positions
      SegIter si = seg_iter(sp);
      int pidx, kt0, kt1, slot, sidx = 0, it = 0;
      while (!aborted && si.next(pidx, kt0, kt1, slot)) {
        const PairInfo pi = pair_info(pidx, p);
        if (sidx > 0 && !warp_wait(&bar[SB_QFREE], (sidx - 1) & 1, lim)) { fail(p, aborted); break; }
        if (lane == 0) {
          mbar_expect_tx(&bar[SB_Q], 2 * kTileBytes);
          tma_load_3d(smem + OFF_QA, &q_map, &bar[SB_Q], 0, pi.i0_a, pi.bhq_a);
          tma_load_3d(smem + OFF_QA + kHalfBytes, &q_map, &bar[SB_Q], 64, pi.i0_a, pi.bhq_a);
          tma_load_3d(smem + OFF_QB, &q_map, &bar[SB_Q], 0, pi.i0_b, pi.bhq_b);
          tma_load_3d(smem + OFF_QB + kHalfBytes, &q_map, &bar[SB_Q], 64, pi.i0_b, pi.bhq_b);
          mbar_arrive(&bar[SB_Q]);
        }
        const int32_t *tpg = p.token_pos + (size_t)pi.bg * p.N_C;
        for (int kt = kt0; kt < kt1; ++kt, ++it) {
          const int s = it & 1;
          if (it >= 2 && !warp_wait(&bar[SB_KEMPTY0 + s], ((it >> 1) - 1) & 1, lim)) {
            fail(p, aborted);
            break;
          }
          uint64_t *full = &bar[SB_KFULL0 + s];
          uint8_t *kdst = smem + (s ? OFF_K1 : OFF_K0);
          if (lane == 0) {
            mbar_expect_tx(full, kTileBytes);
            tma_load_3d(kdst, &k_map, full, 0, kt * BN, pi.bg);
            tma_load_3d(kdst + kHalfBytes, &k_map, full, 64, kt * BN, pi.bg);
            if (kt + kPrefetch < kt1) {
              tma_prefetch_l2_3d(&k_map, 0, (kt + kPrefetch) * BN, pi.bg);
              tma_prefetch_l2_3d(&k_map, 64, (kt + kPrefetch) * BN, pi.bg);
            }
          }
          const int nv = min(BN, p.N_C - kt * BN);
          float *rel = reinterpret_cast<float *>(tp_s) + s * BN;
#pragma unroll
          for (int e = lane; e < BN; e += 32) {
            const int64_t t = e < nv ? (int64_t)tpg[kt * BN + e] : (int64_t)kEmptyPos;
            const int64_t r = t - (int64_t)p.P;
            rel[e] = (float)(r < -1 ? -1 : (r > kRelFar ? kRelFar : r));
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(full);
        }
        ++sidx;
      }
      if (lane == 0 && sidx > 0) {
        mbar_wait(&bar[SB_Q], (sidx - 1) & 1, 4000000000ull);
        for (int k = it - 1; k >= 0 && k >= it - 2; --k)
          mbar_wait(&bar[SB_KFULL0 + (k & 1)], (k >> 1) & 1, 4000000000ull);
      }
    } else if (warp == 2) {
      // ------------------------------------------------------------------ V tiles
      if (lane == 0) {
        SegIter si = seg_iter(sp);
        int pidx, kt0, kt1, slot, it = 0;
        while (!aborted && si.next(pidx, kt0, kt1, slot)) {
          const int bg = pidx / p.ctas_per_group;
          for (int kt = kt0; kt < kt1; ++kt, ++it) {
            const int vs = it & 1;
            if (it >= 2 && !mbar_wait(&bar[SB_VEMPTY0 + vs], ((it >> 1) - 1) & 1, lim)) {
              fail(p, aborted);
              break;
            }
            uint8_t *vdst = smem + (vs ? OFF_V1 : OFF_V0);
            mbar_expect_tx(&bar[SB_VFULL0 + vs], kTileBytes);
            tma_load_3d(vdst, &v_map, &bar[SB_VFULL0 + vs], 0, kt * BN, bg);
            tma_load_3d(vdst + kHalfBytes, &v_map, &bar[SB_VFULL0 + vs], 64, kt * BN, bg);
            mbar_arrive(&bar[SB_VFULL0 + vs]);
            if (kt + kPrefetch < kt1) {
              tma_prefetch_l2_3d(&v_map, 0, (kt + kPrefetch) * BN, bg);
              tma_prefetch_l2_3d(&v_map, 64, (kt + kPrefetch) * BN, bg);
            }
          }
        }
        for (int k = it - 1; k >= 0 && k >= it - 2; --k)
          mbar_wait(&bar[SB_VFULL0 + (k & 1)], (k >> 1) & 1, 4000000000ull);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t qa_addr = sbase + OFF_QA, qb_addr = sbase + OFF_QB, p_addr = sbase + OFF_P;
        // S^T_x(it) = K Q_x^T into columns 0 (a) / 128 (b); O_x += P_x V into 256 (a) / 384 (b)
        auto issue_st = [&](int it, bool tile_b) -> bool {
          const int s = it & 1;
          if (!tile_b && !mbar_wait(&bar[SB_KFULL0 + s], (it >> 1) & 1, lim)) return false;
          if (it >= 1 && !mbar_wait(&bar[tile_b ? SB_TFREEB : SB_TFREEA], (it - 1) & 1, lim))
            return false;
          tc_fence_after();
          const uint32_t k_addr = sbase + (s ? OFF_K1 : OFF_K0);
          const uint32_t q_addr = tile_b ? qb_addr : qa_addr;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_bf16_ss(tmem + (tile_b ? 128 : 0), kmajor_desc(k_addr, ks), kmajor_desc(q_addr, ks),
                        IDESC_K_MAJOR, ks > 0);
          mma_commit(&bar[tile_b ? SB_TFULLB : SB_TFULLA]);
          if (tile_b) mma_commit(&bar[SB_KEMPTY0 + s]);
          return true;
        };
        auto issue_pv = [&](int it, bool tile_b, bool first) -> bool {
          if (!mbar_wait(&bar[tile_b ? SB_PFULLB : SB_PFULLA], it & 1, lim)) return false;
          if (!tile_b && !mbar_wait(&bar[SB_VFULL0 + (it & 1)], (it >> 1) & 1, lim)) return false;
          tc_fence_after();
          const uint32_t v_addr = sbase + ((it & 1) ? OFF_V1 : OFF_V0);
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)
            mma_bf16_ss(tmem + (tile_b ? 384 : 256), mnmajor_desc(p_addr, ks),
                        mnmajor_desc(v_addr, ks), IDESC_PV, (!first || ks > 0) ? 1u : 0u);
          mma_commit(&bar[tile_b ? SB_PFREEB : SB_PFREEA]);
          if (tile_b) mma_commit(&bar[SB_VEMPTY0 + (it & 1)]);
          return true;
        };
        SegIter si = seg_iter(sp);
        int pidx, kt0, kt1, slot, sidx = 0, it = 0;
        while (!aborted && si.next(pidx, kt0, kt1, slot)) {
          const int n = kt1 - kt0;
          if (!mbar_wait(&bar[SB_Q], sidx & 1, lim)) { fail(p, aborted); break; }
          // the previous segment's O has been read out of TMEM
          if (sidx > 0 && !mbar_wait(&bar[SB_OFREE], (sidx - 1) & 1, lim)) { fail(p, aborted); break; }
          tc_fence_after();
          bool ok = issue_st(it, false) && issue_st(it, true);
          for (int j = 0; ok && j < n; ++j) {
            if (j + 1 < n) ok = issue_st(it + j + 1, false) && issue_st(it + j + 1, true);
            if (ok && j + 1 == n) mma_commit(&bar[SB_QFREE]);  // no later MMA of this segment reads Q
            if (ok) ok = issue_pv(it + j, false, j == 0) && issue_pv(it + j, true, j == 0);
          }
          if (!ok) { fail(p, aborted); break; }
          mma_commit(&bar[SB_OFULL]);
          it += n;
          ++sidx;
        }
        mma_commit(&bar[SB_DRAIN]);
        mbar_wait(&bar[SB_DRAIN], 0, 4000000000ull);
      }
      __syncwarp();
    }
  } else {
    reg_alloc<kSoftRegs>();
    // ------------------------ per-slot probabilities, sums and epilogue, one warpgroup per tile
    const int wg = (warp - 4) >> 2;
    const int st = threadIdx.x - 128 * (1 + wg);
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const float c2 = p.scale2;
    float *lse_t = lse_s + wg * BM;  // -lse2 of the tile's rows
    const uint32_t p_row = sbase + OFF_P + (st >> 3) * 1024 + (st & 7) * 128;
    SegIter si = seg_iter(sp);
    int pidx, kt0, kt1, slot, sidx = 0, it = 0;
    // every warp of the warpgroup meets the same named barriers in every segment, also
    // after a failed wait (the work is then skipped), so none of them waits forever
    while (si.next(pidx, kt0, kt1, slot)) {
      const PairInfo pi = pair_info(pidx, p);
      const int i0 = wg ? pi.i0_b : pi.i0_a, bhq = wg ? pi.bhq_b : pi.bhq_a, t = wg ? pi.t_b : pi.t_a;
      // the final LSE of row st: combine the pair's partial (max, sum) in CTA order
      const int c_first = cta_of_unit((long long)pidx * p.n_kt, sp);
      const int c_last = cta_of_unit((long long)(pidx + 1) * p.n_kt - 1, sp);
      float m = -INFINITY;
      for (int c = c_first; c <= c_last; ++c)
        m = fmaxf(m, sp.part_ml[((size_t)c * sp.max_seg + seg_slot(pidx, c, sp)) * (2 * BM) + wg * BM + st].x);
      float l = 0.f;
      if (m != -INFINITY)
        for (int c = c_first; c <= c_last; ++c) {
          const float2 ml = sp.part_ml[((size_t)c * sp.max_seg + seg_slot(pidx, c, sp)) * (2 * BM) + wg * BM + st];
          l += ml.y * ex2(ml.x - m);
        }
      const bool seen = l > 0.f && m > -0.5f * kMaskBias;
      const float lse2 = seen ? m + lg2(l) : -INFINITY;
      named_bar_sync(1 + wg, 128);  // the previous segment's reads of lse_t are done
      lse_t[st] = seen ? -lse2 : -kMaskBias;
      if (p.lse_out && kt0 == 0 && i0 + st < p.S)
        p.lse_out[(size_t)bhq * p.S + i0 + st] = lse2 * 0.69314718055994531f;
      named_bar_sync(1 + wg, 128);
      const int rmax = min(BM, p.S - i0);
      float *pw = p.part_w + ((size_t)bhq * p.tiles + t) * p.N_C;
      uint32_t pk[BM / 2];
      for (int kt = kt0; kt < kt1 && !aborted; ++kt, ++it) {
        const int s = it & 1;
        const int j = kt * BN + st;
        if (!warp_wait(&bar[wg ? SB_TFULLB : SB_TFULLA], it & 1, lim)) { fail(p, aborted); break; }
        if (!warp_wait(&bar[SB_KFULL0 + s], (it >> 1) & 1, lim)) { fail(p, aborted); break; }
        tc_fence_after();
        const float relj = __int_as_float(tp_s[s * BN + st]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[SB_KEMPTY0 + s]);
        const float rmf = fminf(fmaxf(relj - (float)i0, 0.f), (float)BM);
        const int rmin = (int)rmf;
        const bool full = __all_sync(0xffffffffu, rmin == 0 && rmax == BM);
        uint32_t r[BM];
        tmem_ld128(tmem + lane_base + wg * 128, r);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[wg ? SB_TFREEB : SB_TFREEA]);
        const float cs = slot_probs(r, lse_t, c2, rmin, rmax, full, pk);
        // the single P buffer goes a(it) -> b(it) -> a(it + 1)
        bool ok = true;
        if (wg == 1)
          ok = warp_wait(&bar[SB_PFREEA], it & 1, lim);
        else if (it > 0)
          ok = warp_wait(&bar[SB_PFREEB], (it - 1) & 1, lim);
        if (!ok) { fail(p, aborted); break; }
        store_p(p_row, st, pk);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[wg ? SB_PFULLB : SB_PFULLA]);
        if (j < p.N_C) pw[j] = cs;
      }
      // epilogue of the segment: y, or this segment's share of O when the pair is split
      if (!aborted && !warp_wait(&bar[SB_OFULL], sidx & 1, lim)) fail(p, aborted);
      if (aborted) {
        ++sidx;
        continue;
      }
      tc_fence_after();
      const bool whole = kt0 == 0 && kt1 == p.n_kt;
      const int row_i = i0 + st;
      __nv_bfloat16 *yrow = p.y + ((size_t)bhq * p.S + row_i) * D;
      float *orow = sp.part_o + ((((size_t)blockIdx.x * sp.max_seg + slot) * 2 + wg) * BM + st) * D;
      uint32_t o32[32];
#pragma unroll
      for (int cq = 0; cq < 4; ++cq) {
        tmem_ld32(tmem + lane_base + 256 + wg * 128 + cq * 32, o32);
        tmem_wait_ld();
        if (whole) {
          if (row_i < p.S) {
            uint32_t o[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              o[e] = pack_bf16x2(__uint_as_float(o32[2 * e]), __uint_as_float(o32[2 * e + 1]));
            uint4 *dst = reinterpret_cast<uint4 *>(yrow + cq * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
          }
        } else {
          uint4 *dst = reinterpret_cast<uint4 *>(orow + cq * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_uint4(o32[4 * e], o32[4 * e + 1], o32[4 * e + 2], o32[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[SB_OFREE]);
      ++sidx;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// y of the pairs whose slots were split over several CTAs: the sum of their partial
// O rows in CTA order.  One thread per 4 columns of one row (pair, tile, row, column
// group), so that every load of the pass is in flight at once.
__global__ void __launch_bounds__(256)
    reduce_o_kernel(const SplitParams sp, int n_pairs) {
  const TcParams &p = sp.t;
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long per_pair = 2LL * BM * (D / 4);
  const int pidx = (int)(e / per_pair);
  if (pidx >= n_pairs) return;
  const int rem = (int)(e - (long long)pidx * per_pair);
  const int wg = rem / (BM * (D / 4));
  const int row = (rem / (D / 4)) % BM, c4 = rem % (D / 4);
  const int c_first = cta_of_unit((long long)pidx * p.n_kt, sp);
  const int c_last = cta_of_unit((long long)(pidx + 1) * p.n_kt - 1, sp);
  if (c_first == c_last) return;  // written by its only CTA
  const PairInfo pi = pair_info(pidx, p);
  const int i0 = wg ? pi.i0_b : pi.i0_a, bhq = wg ? pi.bhq_b : pi.bhq_a;
  if (i0 + row >= p.S) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c = c_first; c <= c_last; ++c) {
    const float4 v = __ldcs(reinterpret_cast<const float4 *>(
        sp.part_o + ((((size_t)c * sp.max_seg + seg_slot(pidx, c, sp)) * 2 + wg) * BM + row) * D) + c4);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  __nv_bfloat162 *dst =
      reinterpret_cast<__nv_bfloat162 *>(p.y + ((size_t)bhq * p.S + i0 + row) * D + c4 * 4);
  dst[0] = __floats2bfloat162_rn(acc.x, acc.y);
  dst[1] = __floats2bfloat162_rn(acc.z, acc.w);
}

// w[b, g, j] = sum over the group's heads and row tiles of the partial sums;
// wq[b, h, j] = sum over the head's row tiles.  Fixed summation order.
__global__ void __launch_bounds__(256)
    reduce_w_kernel(const float *__restrict__ part_w, float *__restrict__ w,
                    float *__restrict__ wq, int Hq, int Hk, int q_g, int N_C, int tiles,
                    int tiles_used, int n_cols) {
  const int bg = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= N_C) return;
  const int b = bg / Hk, g = bg - b * Hk;
  if (j >= n_cols) {  // slots past the scanned span are empty: no weight
    for (int hl = 0; hl < q_g && wq; ++hl) wq[(size_t)(b * Hq + g * q_g + hl) * N_C + j] = 0.f;
    w[(size_t)bg * N_C + j] = 0.f;
    return;
  }
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

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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


int ensure_cache_maps(h2okv_cache *c) {
  if (c->tc.maps_ready) return H2OKV_OK;
  const h2okv_cache_desc &d = c->desc;
  if (d.kv_dtype != H2OKV_BF16) {  // codes are read with plain loads: no maps for the cache
    memset(c->tc.k_map, 0, sizeof(c->tc.k_map));
    memset(c->tc.v_map, 0, sizeof(c->tc.v_map));
  } else {
    int rc = encode_rows_map(reinterpret_cast<CUtensorMap *>(c->tc.k_map), c->bufs.keys,
                             (uint64_t)d.capacity, (uint64_t)d.batch * d.n_kv_heads);
    if (rc) return rc;
    rc = encode_rows_map(reinterpret_cast<CUtensorMap *>(c->tc.v_map), c->bufs.values,
                         (uint64_t)d.capacity, (uint64_t)d.batch * d.n_kv_heads);
    if (rc) return rc;
  }
  c->tc.maps_ready = true;
  return H2OKV_OK;
}

bool tc_path_supported(const h2okv_cache_desc &d) {
  return d.head_dim == D && d.q_dtype == H2OKV_BF16 &&
         (d.kv_dtype == H2OKV_BF16 || d.kv_dtype == H2OKV_I8 || d.kv_dtype == H2OKV_I4);
}

namespace {
// Split scheduling pays when one CTA per pair of query tiles leaves many SMs idle in
// the last wave (measured: a wave 86 % full runs as fast fused as split, since the
// split kernels cost ~10 % more per unit); it needs two query tiles in every pair and
// a few tiles per CTA.
constexpr double kSplitFill = 0.75;
struct SplitShape {
  bool use;
  long long U;
  int max_seg;
};
SplitShape split_shape(const h2okv_cache_desc &d, int S, int G) {
  SplitShape r{false, 0, 0};
  if (G <= 0 || d.kv_dtype != H2OKV_BF16) return r;
  const int tiles = (S + BM - 1) / BM;
  const int n_qt = (d.n_q_heads / d.n_kv_heads) * tiles;
  if (n_qt % 2) return r;
  const long long pairs = (long long)d.batch * d.n_kv_heads * (n_qt / 2);
  const int n_kt = (d.capacity + BN - 1) / BN;
  r.U = pairs * n_kt;
  const long long waves = (pairs + G - 1) / G;
  const double fill = (double)pairs / (double)(waves * G);
  if (fill >= kSplitFill || r.U < 4LL * G || n_kt < 4) return r;
  const long long per = (r.U + G - 1) / G;  // units of one CTA at most
  r.max_seg = (int)((per + n_kt - 1) / n_kt) + 1;
  r.use = true;
  return r;
}
}  // namespace

void tc_plan(const h2okv_cache_desc &d, TcPlan *plan) {
  plan->enabled = tc_path_supported(d);
  plan->tiles_per_head = (d.max_chunk + BM - 1) / BM;
  plan->split_ctas = 0;
  plan->max_seg = 0;
  // bf16 caches: attention and score sums as two passes unless H2OKV_TC_FUSED=1 selects
  // the single kernel that runs both phases per CTA
  const char *fused = getenv("H2OKV_TC_FUSED");
  plan->two_pass = !(fused && fused[0] == '1');
  int dev = 0, sms = 0;
  plan->sms = 0;
  if (plan->enabled && cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) {
    plan->sms = sms;
    const SplitShape sh = split_shape(d, d.max_chunk, sms);
    if (sh.use) {
      plan->split_ctas = sms;
      plan->max_seg = sh.max_seg;
    }
    if (d.kv_dtype == H2OKV_BF16 && plan->two_pass) {
      // pass 1 on every SM: a CTA holds at most ceil(pairs / SMs) + 2 segments
      const long long pairs = (long long)d.batch * d.n_kv_heads *
                              (((d.n_q_heads / d.n_kv_heads) * plan->tiles_per_head + 1) / 2);
      plan->split_ctas = sms;
      plan->max_seg = max(plan->max_seg, (int)((pairs + sms - 1) / sms) + 2);
    }
  }
  cudaGetLastError();  // a failed query (no device) is not an error here
}

namespace {

// Shared-memory opt-in and the register-allotment check, once per device and dtype.
template <int KV>
int prepare_kernel() {
  static thread_local int ready_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (ready_dev == dev) return H2OKV_OK;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<KV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(attn_tc_kernel): %s",
                     cudaGetErrorString(e));
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_tc_kernel<KV>);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaFuncGetAttributes(attn_tc_kernel): %s",
                     cudaGetErrorString(e));
  // the in-kernel register split assumes exactly this launch allotment
  if (fa.numRegs != launch_regs_of<KV>())
    return set_error(H2OKV_ERR_UNSUPPORTED,
                     "attn_tc_kernel built with %d registers per thread, expected %d", fa.numRegs,
                     launch_regs_of<KV>());
  ready_dev = dev;
  return H2OKV_OK;
}

// The same set-up for a split kernel.
template <typename K>
int prepare_split_kernel(K kernel, int &ready_dev, const char *name) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (ready_dev == dev) return H2OKV_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(%s): %s", name, cudaGetErrorString(e));
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaFuncGetAttributes(%s): %s", name, cudaGetErrorString(e));
  if (fa.numRegs != kLaunchRegs)
    return set_error(H2OKV_ERR_UNSUPPORTED, "%s built with %d registers per thread, expected %d",
                     name, fa.numRegs, kLaunchRegs);
  ready_dev = dev;
  return H2OKV_OK;
}

// Shared-memory opt-in and register check of a bf16 two-pass kernel.
template <typename K>
int prepare_pass_kernel(K kernel, uint32_t smem_bytes, int regs, int &ready_dev, const char *name) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (ready_dev == dev) return H2OKV_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_bytes);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaFuncSetAttribute(%s): %s", name, cudaGetErrorString(e));
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess)
    return set_error(H2OKV_ERR_CUDA, "cudaFuncGetAttributes(%s): %s", name, cudaGetErrorString(e));
  if (fa.numRegs != regs)
    return set_error(H2OKV_ERR_UNSUPPORTED, "%s built with %d registers per thread, expected %d",
                     name, fa.numRegs, regs);
  ready_dev = dev;
  return H2OKV_OK;
}

template <int KV>
int launch_kernel(int grid, const CUtensorMap &qmap, const CUtensorMap &kmap,
                  const CUtensorMap &vmap, const TcParams &prm, cudaStream_t st) {
  int rc = prepare_kernel<KV>();
  if (rc) return rc;
  attn_tc_kernel<KV><<<grid, threads_of<KV>(), kSmemBytes, st>>>(qmap, kmap, vmap, prm);
  return check_launch("attn_tc_kernel");
}

}  // namespace

int launch_attn_tc(h2okv_cache *c, const void *q, int S, int64_t P, void *y, float *lse, float *w,
                   float *wq, cudaStream_t st) {
  const h2okv_cache_desc &d = c->desc;
  uint8_t *ws = reinterpret_cast<uint8_t *>(c->bufs.workspace);
  int rc = ensure_cache_maps(c);
  if (rc) return rc;
  CUtensorMap qmap;
  rc = encode_rows_map(&qmap, q, (uint64_t)S, (uint64_t)d.batch * d.n_q_heads);
  if (rc) return rc;

  TcParams prm;
  prm.token_pos = c->bufs.token_pos;
  prm.kq = reinterpret_cast<const uint8_t *>(c->bufs.keys);
  prm.vq = reinterpret_cast<const uint8_t *>(c->bufs.values);
  prm.ksc = reinterpret_cast<const __half *>(c->bufs.k_scales);
  prm.vsc = reinterpret_cast<const __half *>(c->bufs.v_scales);
  prm.y = reinterpret_cast<__nv_bfloat16 *>(y);
  prm.lse_out = lse;
  prm.part_w = reinterpret_cast<float *>(ws + c->ws.part_w);
  prm.nlse = reinterpret_cast<float *>(ws + c->ws.nlse);
  prm.status = reinterpret_cast<int *>(ws + c->ws.status);
  prm.Hq = d.n_q_heads;
  prm.Hk = d.n_kv_heads;
  prm.q_g = d.n_q_heads / d.n_kv_heads;
  prm.N_C = d.capacity;
  prm.S = S;
  prm.P = (int)P;
  prm.tiles = (S + BM - 1) / BM;
  prm.n_kt = (d.capacity + BN - 1) / BN;
  int n_cols = d.capacity;  // slots whose weights the kernels write
  prm.ctas_per_group = (prm.q_g * prm.tiles + 1) / 2;
  prm.scale2 = (float)(1.4426950408889634 / 11.313708498984761);  // log2(e) / sqrt(128)
  prm.timeout_ns = c->wait_timeout_ns;
  const int grid = d.batch * d.n_kv_heads * prm.ctas_per_group;
  const CUtensorMap &kmap = *reinterpret_cast<const CUtensorMap *>(c->tc.k_map);
  const CUtensorMap &vmap = *reinterpret_cast<const CUtensorMap *>(c->tc.v_map);
  // split scheduling: every SM gets the same share of (pair, K/V tile) units
  const SplitShape sh = split_shape(d, S, c->tc.split_ctas);
  // (the fused kernel's split schedule; the two-pass path splits its own work)
  if (sh.use && sh.max_seg <= c->tc.max_seg && !(d.kv_dtype == H2OKV_BF16 && c->tc.two_pass)) {
    static thread_local int ready_a = -1, ready_b = -1;
    rc = prepare_split_kernel(attn_split_a_kernel, ready_a, "attn_split_a_kernel");
    if (rc) return rc;
    rc = prepare_split_kernel(attn_split_b_kernel, ready_b, "attn_split_b_kernel");
    if (rc) return rc;
    SplitParams sp;
    sp.t = prm;
    sp.G = c->tc.split_ctas;
    sp.max_seg = c->tc.max_seg;
    sp.U = sh.U;
    sp.part_ml = reinterpret_cast<float2 *>(ws + c->ws.part_ml);
    sp.part_o = reinterpret_cast<float *>(ws + c->ws.part_o);
    attn_split_a_kernel<<<sp.G, kThreads, kSmemBytes, st>>>(qmap, kmap, sp);
    rc = check_launch("attn_split_a_kernel");
    if (rc) return rc;
    attn_split_b_kernel<<<sp.G, kThreads, kSmemBytes, st>>>(qmap, kmap, vmap, sp);
    rc = check_launch("attn_split_b_kernel");
    if (rc) return rc;
    const int n_pairs = grid;
    const long long n_threads = (long long)n_pairs * 2 * BM * (D / 4);
    reduce_o_kernel<<<(unsigned)((n_threads + 255) / 256), 256, 0, st>>>(sp, n_pairs);
    rc = check_launch("reduce_o_kernel");
    if (rc) return rc;
    dim3 rgrid((d.capacity + 255) / 256, d.batch * d.n_kv_heads);
    reduce_w_kernel<<<rgrid, 256, 0, st>>>(prm.part_w, w, wq, d.n_q_heads, d.n_kv_heads, prm.q_g,
                                           d.capacity, prm.tiles, prm.tiles, n_cols);
    return check_launch("reduce_w_kernel");
  }
  // outside the split schedule the kernels scan only the K/V tiles that may hold an
  // occupied slot (the cache fills left to right)
  prm.n_kt = (max(c->n_span, 1) + BN - 1) / BN;
  n_cols = min(d.capacity, prm.n_kt * BN);
  if (d.kv_dtype == H2OKV_BF16 && c->tc.two_pass) {
    // attention with an online softmax, then the score sums against the final LSE
    static thread_local int ready_f = -1, ready_s = -1;
    rc = prepare_pass_kernel(attn_fwd_kernel, kSmemF, kLaunchRegs, ready_f, "attn_fwd_kernel");
    if (rc) return rc;
    rc = prepare_pass_kernel(scoresum_kernel, kSmemS, kLaunchRegsS, ready_s, "scoresum_kernel");
    if (rc) return rc;
    // attention over equal shares of (pair, K/V tile) units, one CTA per SM when the
    // partial-result workspace holds every CTA's pieces, else one CTA per pair
    SplitParams fs{};
    fs.t = prm;
    fs.U = (long long)grid * prm.n_kt;
    fs.G = grid;
    fs.max_seg = c->tc.max_seg;
    fs.part_ml = reinterpret_cast<float2 *>(ws + c->ws.part_ml);
    fs.part_o = reinterpret_cast<float *>(ws + c->ws.part_o);
    const int G = (int)min((long long)c->tc.split_ctas, fs.U);
    // Only when one CTA per pair leaves over a quarter of the SMs idle in the last wave,
    // and the scan is long: otherwise the partial results' round trip and the K/V
    // tiles that CTAs of a group no longer share in L2 cost more than the idle SMs.
    const int sms = max(c->tc.sms, 1);
    const double fill = (double)grid / (double)(((grid + sms - 1) / sms) * sms);
    if (G > grid && prm.n_kt >= kMinSplitTiles && fill < kSplitFill) {
      const long long per = (fs.U + G - 1) / G;
      const long long segs = (per + prm.n_kt - 1) / prm.n_kt + 1;
      // a pair spans at most ceil(n_kt / (per - 1)) + 1 CTAs
      const long long pieces = per > 1 ? (prm.n_kt + per - 2) / (per - 1) + 1 : prm.n_kt;
      if (segs <= c->tc.max_seg && segs <= kMaxSegF && pieces <= kMaxPieces) fs.G = G;
    }
    attn_fwd_kernel<<<fs.G, kThreads, kSmemF, st>>>(qmap, kmap, vmap, fs);
    rc = check_launch("attn_fwd_kernel");
    if (rc) return rc;
    if (fs.G != grid) {
      combine_fwd_kernel<<<dim3(grid, 2 * BM * (D / 4) / 256), 256, 0, st>>>(fs);
      rc = check_launch("combine_fwd_kernel");
      if (rc) return rc;
    }
    // the score sums over equal shares of (pair, K tile) units, one CTA per SM
    SplitParams ss{};
    ss.t = prm;
    ss.U = (long long)grid * prm.n_kt;
    ss.G = (int)min((long long)max(c->tc.sms, 1), ss.U);
    scoresum_kernel<<<ss.G, kThreadsS, kSmemS, st>>>(qmap, kmap, ss);
    rc = check_launch("scoresum_kernel");
    if (rc) return rc;
    dim3 rgrid((d.capacity + 255) / 256, d.batch * d.n_kv_heads);
    reduce_w_kernel<<<rgrid, 256, 0, st>>>(prm.part_w, w, wq, d.n_q_heads, d.n_kv_heads, prm.q_g,
                                           d.capacity, prm.tiles, prm.tiles, n_cols);
    return check_launch("reduce_w_kernel");
  }
  switch (d.kv_dtype) {
    case H2OKV_BF16: rc = launch_kernel<H2OKV_BF16>(grid, qmap, kmap, vmap, prm, st); break;
    case H2OKV_I8: rc = launch_kernel<H2OKV_I8>(grid, qmap, kmap, vmap, prm, st); break;
    case H2OKV_I4: rc = launch_kernel<H2OKV_I4>(grid, qmap, kmap, vmap, prm, st); break;
    default: return set_error(H2OKV_ERR_UNSUPPORTED, "kv dtype on the tensor-core path");
  }
  if (rc) return rc;
  dim3 rgrid((d.capacity + 255) / 256, d.batch * d.n_kv_heads);
  reduce_w_kernel<<<rgrid, 256, 0, st>>>(prm.part_w, w, wq, d.n_q_heads, d.n_kv_heads, prm.q_g,
                                         d.capacity, prm.tiles, prm.tiles, n_cols);
  return check_launch("reduce_w_kernel");
}

}  // namespace h2okv
