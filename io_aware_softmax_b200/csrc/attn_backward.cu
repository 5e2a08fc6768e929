// Backward pass of the fused attention for sm_100a: dQ, dK, dV from (Q, K, V, O, dO, LSE)
// without any N x N matrix in memory.  S and P are recomputed tile by tile from the saved
// row log-sum-exp -- the recomputation strategy of "FlashAttention 논문 분석: IO-Aware Exact
// Attention" (sections "FlashAttention v1: Tiling + Recomputation" and "Recomputation 전략")
// -- and the gradients are the calculus of the definition:
//   P = exp(scale q.k - LSE),  dP = dO V^T,  D = rowsum(dO * O),  dS = P (dP - D),
//   dV = P^T dO,  dQ = scale dS K,  dK = scale dS^T Q   (GQA: dK, dV sum over the group).
//
// Three launches:
//   * attn_bwd_rowdot_kernel: D and the base-2 LSE of every query row (one warp per row);
//   * attn_bwd_dq_kernel: one CTA per 128-row query tile; the K/V tiles its rows can see
//     stream through a TMA ring; per K/V tile the tensor core computes S = Q K^T and
//     dP = dO V^T into two TMEM buffers, a warpgroup (thread r = row r) turns them into
//     bf16 dS written back into the low half of the dP buffer, and the tensor core adds
//     dS K (A read from TMEM, K as an MN-major operand) into the dQ accumulator in TMEM;
//   * attn_bwd_dkdv_kernel: one CTA per 128-key tile of a KV head; the (Q, dO) tiles of
//     every query head of its group that can see the keys stream through the ring; the
//     tensor core computes S^T = K Q^T and dP^T = V dO^T, the warpgroup (thread r = key r)
//     writes bf16 P^T and dS^T into the low halves of those buffers, and dV += P^T dO and
//     dK += dS^T Q accumulate in TMEM -- dK and dV of a tile are complete in one CTA, so
//     nothing is accumulated with atomics.
// Warps: 0-7 two element-wise warpgroups (group g owns the tile's columns [64g, 64g + 64)
// in every TMEM lane), 8 the tcgen05 issuer (whole warp, elect.sync), 9 the TMA producer,
// 10-11 the per-query vectors of the streamed tiles (key-tile kernel; idle in the query-tile
// kernel).  Warps 8-11 give registers to the element-wise groups with setmaxnreg.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "attn_internal.h"
#include "mask.cuh"
#include "sm100_ptx.cuh"
#include "tmem_ldst.cuh"

namespace attn {

namespace {

constexpr int kBT = 128;                 // rows of every tile (queries or keys)
constexpr int kBwdThreads = 384;
constexpr int kBwdMmaWarp = 8;
constexpr int kBwdTmaWarp = 9;
// setmaxnreg split of the 384 x 168 launch registers: 2 x 128 x 200 + 128 x 104 = 64512
constexpr uint32_t kBwdRegsElem = 200;
constexpr uint32_t kBwdRegsOther = 104;
constexpr float kLog2eB = 1.44269504088896341f;
constexpr uint32_t kTmemX = 0;           // S or S^T (fp32), then bf16 P^T (see below)
constexpr uint32_t kTmemY = 128;         // dP or dP^T (fp32), then bf16 dS / dS^T
// The bf16 result of fp32 columns [64g, 64g + 64) goes to columns [64g, 64g + 32) of the same
// buffer: each warpgroup overwrites only columns it has already read itself, so the two
// groups never wait for each other.  Contraction step kk (16 columns) then sits at TMEM
// column 8 kk, plus 32 for the second group's half.
constexpr uint32_t kTmemAcc0 = 256;      // dQ, or dV
constexpr uint32_t kTmemAcc1 = 384;      // dK

template <int D>
struct BwdCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kChunkBytes = kBT * 128;
  static constexpr int kTileBytes = kBT * D * 2;
  static constexpr int kStages = (D == 128) ? 2 : 4;     // ring stages of two tiles each
  static constexpr int kStatOff = 0;                     // two stationary tiles
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kVecOff = kRingOff + kStages * 2 * kTileBytes;
  static constexpr int kVecBytes = 2 * 4 * kBT * 4;      // [2 parities][lse2, D, lo, hi][128]
  static constexpr int kBarOff = kVecOff + kVecBytes;
  // stat, full[S], empty[S], s_ready, dp_ready, p_ready (or x_free), ds_ready, acc, done,
  // vec_full[2], vec_empty[2]
  static constexpr int kNumBars = 11 + 2 * kStages;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;
};

// The query-tile kernel streams K and V through separate rings: a K tile is read by S = Q K^T
// (issued as soon as the previous S is in registers) and by dQ += dS K at the end of its
// step, so it lives about two steps and gets three slots; a V tile is read only by
// dP = dO V^T and gets two.  The early S of the next tile then never waits for its K.
template <int D>
struct DqCfg {
  static constexpr int kTileBytes = BwdCfg<D>::kTileBytes;
  static constexpr int kSlotsK = 3, kSlotsV = 2;
  static constexpr int kStatOff = 0;                     // Q and dO of the CTA's query tile
  static constexpr int kKOff = 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kSlotsK * kTileBytes;
  static constexpr int kBarOff = kVOff + kSlotsV * kTileBytes;
  // stat, fullK[3], emptyK[3], fullV[2], emptyV[2], s, dp, x_free, ds, acc, done
  static constexpr int kFullK = 1, kEmptyK = 1 + kSlotsK, kFullV = 1 + 2 * kSlotsK,
                       kEmptyV = 1 + 2 * kSlotsK + kSlotsV, kOwn = 1 + 2 * (kSlotsK + kSlotsV);
  static constexpr int kNumBars = kOwn + 6;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;
};

enum : uint32_t {
  kSiteBwdStat = 201, kSiteBwdFull, kSiteBwdEmpty, kSiteBwdS, kSiteBwdP, kSiteBwdAcc,
  kSiteBwdDrain, kSiteBwdVecFull, kSiteBwdVecEmpty,
};

__device__ __forceinline__ float bf(uint32_t u) { return __uint_as_float(u); }

// The two element-wise steps of the recomputed tile for one TMEM lane, four columns at a
// time (column groups j = 0 .. N/4 - 1 of the loaded run):
//   probs: s (raw q.k, fp32 bits) becomes p = 2^(s ks - l2), 0 where vis(j) has no bit;
//   grads: ds = p (dp - Dv) and bf16 pairs of ds (and of p, optionally) for the 32 columns
//          [OFF, OFF + 32).
// l2(j) and dv(j) give the four columns' values, vis(j) a 4-bit mask of visible pairs.
// kCap: the score is soft-capped, x = cap_log2 tanh(s cap_scale) - l2 (base 2).  When every
// raw score of the run, in every lane of the warp, lies in the polynomial's range
// (|s| <= cap_fast_max), x is the polynomial of cap_poly with the subtraction folded into
// its last step -- square, four Horner multiply-adds and one more, in paired f32x2
// instructions, no MUFU work besides the exponential; otherwise tanh(y) = 1 - 2/(e^(2y)+1)
// on ex2 and rcp.  The choice is per warp and per call, so the loop that runs is one
// straight block of code.
// kKeepX (with kCap): s keeps the base-2 exponent x itself (-inf where not visible) instead
// of p = 2^x, for a caller whose grads step takes kFromX.
template <int N, bool kCap = false, bool kKeepX = false, typename L2, typename Vis>
__device__ __forceinline__ void probs(uint32_t (&s)[N], float ks, L2 l2, Vis vis,
                                      const BwdParams& bp) {
  static_assert(!kKeepX || kCap, "the exponent is kept on the soft-cap path only");
  if constexpr (kCap) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int c = 0; c < N; c += 4) {
      a0 = max3f(a0, fabsf(bf(s[c])), fabsf(bf(s[c + 1])));
      a1 = max3f(a1, fabsf(bf(s[c + 2])), fabsf(bf(s[c + 3])));
    }
    if (__all_sync(0xffffffffu, fmaxf(a0, a1) <= bp.cap_fast_max)) {
      const float b0 = bp.cap_poly[0], b1 = bp.cap_poly[1], b2 = bp.cap_poly[2],
                  b3 = bp.cap_poly[3], b4 = bp.cap_poly[4];
#pragma unroll
      for (int j = 0; j < N / 4; ++j) {
        const float4 l = l2(j);
        const unsigned m = vis(j);
        const int c = 4 * j;
        float x[4];
#pragma unroll
        for (int h = 0; h < 4; h += 2) {
          const float s0 = bf(s[c + h]), s1 = bf(s[c + h + 1]);
          float w0, w1, t0, t1;
          fmul2(w0, w1, s0, s1, s0, s1);
          ffma2(t0, t1, w0, w1, b4, b4, b3, b3);
          ffma2(t0, t1, t0, t1, w0, w1, b2, b2);
          ffma2(t0, t1, t0, t1, w0, w1, b1, b1);
          ffma2(t0, t1, t0, t1, w0, w1, b0, b0);
          ffma2(x[h], x[h + 1], t0, t1, s0, s1, h ? -l.z : -l.x, h ? -l.w : -l.y);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
          s[c + i] = __float_as_uint(((m >> i) & 1u) ? (kKeepX ? x[i] : ex2_approx(x[i]))
                                                     : (kKeepX ? -INFINITY : 0.f));
      }
      return;
    }
  }
#pragma unroll
  for (int j = 0; j < N / 4; ++j) {
    const float4 l = l2(j);
    const unsigned m = vis(j);
    const int c = 4 * j;
    float x0, x1, x2, x3;
    if constexpr (kCap) {
      x0 = fmaf(bp.cap_log2, tanh_via_ex2(bf(s[c]) * bp.cap_scale), -l.x);
      x1 = fmaf(bp.cap_log2, tanh_via_ex2(bf(s[c + 1]) * bp.cap_scale), -l.y);
      x2 = fmaf(bp.cap_log2, tanh_via_ex2(bf(s[c + 2]) * bp.cap_scale), -l.z);
      x3 = fmaf(bp.cap_log2, tanh_via_ex2(bf(s[c + 3]) * bp.cap_scale), -l.w);
    } else {
      ffma2(x0, x1, bf(s[c]), bf(s[c + 1]), ks, ks, -l.x, -l.y);
      ffma2(x2, x3, bf(s[c + 2]), bf(s[c + 3]), ks, ks, -l.z, -l.w);
    }
    if constexpr (kKeepX) {
      s[c] = __float_as_uint((m & 1u) ? x0 : -INFINITY);
      s[c + 1] = __float_as_uint((m & 2u) ? x1 : -INFINITY);
      s[c + 2] = __float_as_uint((m & 4u) ? x2 : -INFINITY);
      s[c + 3] = __float_as_uint((m & 8u) ? x3 : -INFINITY);
    } else {
      s[c] = __float_as_uint((m & 1u) ? ex2_approx(x0) : 0.f);
      s[c + 1] = __float_as_uint((m & 2u) ? ex2_approx(x1) : 0.f);
      s[c + 2] = __float_as_uint((m & 4u) ? ex2_approx(x2) : 0.f);
      s[c + 3] = __float_as_uint((m & 8u) ? ex2_approx(x3) : 0.f);
    }
  }
}

// With a soft-cap (kCap) the capped score y = c tanh(x / c) passes dy (1 - tanh^2) on to the
// scaled product x; tanh is recovered from p itself, t = (log2 p + l2) / cap_log2, so no
// register holds it between the two steps (p = 0 leaves ds = 0 whatever the factor).
__device__ __forceinline__ float cap_factor(float p, float l, float inv_cap_log2) {
  const float t = (p > 0.f) ? (__log2f(p) + l) * inv_cap_log2 : 0.f;
  return fmaf(-t, t, 1.f);
}

// kFromX (with kCap): pr holds the base-2 exponents x of probs<..., kKeepX>; p = 2^x here,
// and tanh = (x + l2) / cap_log2 comes from x directly, so the pair of steps takes one MUFU
// operation per score (the exponential) instead of an exponential and a logarithm.
__device__ __forceinline__ float cap_factor_x(float x, float l, float inv_cap_log2) {
  const float t = (x + l) * inv_cap_log2;
  return (x != -INFINITY) ? fmaf(-t, t, 1.f) : 0.f;
}

template <bool kWantP, int OFF, int N, int ND, bool kCap = false, bool kFromX = false,
          typename DV, typename L2 = float4 (*)(int)>
__device__ __forceinline__ void grads(const uint32_t (&pr)[N], const uint32_t (&dp)[ND], DV dv,
                                      uint32_t (&pk)[16], uint32_t (&dsk)[16], L2 l2 = nullptr,
                                      float inv_cap_log2 = 0.f) {
  static_assert(ND == 32 || ND == N, "dp holds these 32 columns or all N");
  static_assert(!kFromX || kCap, "exponents are kept on the soft-cap path only");
  constexpr int DOFF = (ND == 32) ? 0 : OFF;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 d = dv(j);
    const int c = OFF + 4 * j, e = DOFF + 4 * j;
    float p0, p1, p2, p3;
    if constexpr (kFromX) {
      p0 = ex2_approx(bf(pr[c]));
      p1 = ex2_approx(bf(pr[c + 1]));
      p2 = ex2_approx(bf(pr[c + 2]));
      p3 = ex2_approx(bf(pr[c + 3]));
    } else {
      p0 = bf(pr[c]);
      p1 = bf(pr[c + 1]);
      p2 = bf(pr[c + 2]);
      p3 = bf(pr[c + 3]);
    }
    float d0 = p0 * (bf(dp[e]) - d.x);
    float d1 = p1 * (bf(dp[e + 1]) - d.y);
    float d2 = p2 * (bf(dp[e + 2]) - d.z);
    float d3 = p3 * (bf(dp[e + 3]) - d.w);
    if constexpr (kCap && kFromX) {
      const float4 l = l2(j);
      d0 *= cap_factor_x(bf(pr[c]), l.x, inv_cap_log2);
      d1 *= cap_factor_x(bf(pr[c + 1]), l.y, inv_cap_log2);
      d2 *= cap_factor_x(bf(pr[c + 2]), l.z, inv_cap_log2);
      d3 *= cap_factor_x(bf(pr[c + 3]), l.w, inv_cap_log2);
    } else if constexpr (kCap) {
      const float4 l = l2(j);
      d0 *= cap_factor(p0, l.x, inv_cap_log2);
      d1 *= cap_factor(p1, l.y, inv_cap_log2);
      d2 *= cap_factor(p2, l.z, inv_cap_log2);
      d3 *= cap_factor(p3, l.w, inv_cap_log2);
    }
    if (kWantP) {
      pk[2 * j] = pack_bf16x2(p0, p1);
      pk[2 * j + 1] = pack_bf16x2(p2, p3);
    }
    dsk[2 * j] = pack_bf16x2(d0, d1);
    dsk[2 * j + 1] = pack_bf16x2(d2, d3);
  }
}

// bf16 pairs of 32 fp32 values.
__device__ __forceinline__ void pack_pairs(const uint32_t (&v)[32], uint32_t (&pk)[16]) {
#pragma unroll
  for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(bf(v[2 * k]), bf(v[2 * k + 1]));
}

// First / last query row whose visible key interval meets keys [k0, k1] (the intervals are
// non-decreasing at both ends, so the rows that see the tile form one range); qa > qb when
// no row does.
__device__ __forceinline__ void query_range(const MaskParams& m, int Nq, int k0, int k1, int& qa,
                                            int& qb) {
  int lo = 0, hi = Nq;             // first row with hi(q) >= k0
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    int a, b;
    row_interval(m, mid, a, b);
    if (b >= k0) hi = mid; else lo = mid + 1;
  }
  qa = lo;
  lo = -1;
  hi = Nq - 1;                     // last row with lo(q) <= k1
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    int a, b;
    row_interval(m, mid, a, b);
    if (a <= k1) lo = mid; else hi = mid - 1;
  }
  qb = lo;
}

// One row of NCOL fp32 TMEM columns (read in 32-column chunks), times mul, rounded to bf16
// and written to global memory when the row exists.
template <int NCOL>
__device__ __forceinline__ void store_row(uint32_t taddr, float mul, __nv_bfloat16* dst,
                                          bool valid) {
#pragma unroll
  for (int cc = 0; cc < NCOL / 32; ++cc) {
    uint32_t a[32];
    tmem_ld_x32(taddr + 32u * cc, a);
    uint32_t wv[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) wv[k] = pack_bf16x2(bf(a[2 * k]) * mul, bf(a[2 * k + 1]) * mul);
    if (valid) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cc);
#pragma unroll
      for (int k = 0; k < 4; ++k) d4[k] = make_uint4(wv[4 * k], wv[4 * k + 1], wv[4 * k + 2],
                                                      wv[4 * k + 3]);
    }
  }
}

__device__ __forceinline__ void store_zero_row(__nv_bfloat16* dst, int n, bool valid) {
  if (!valid) return;
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  for (int k = 0; k < n / 8; ++k) d4[k] = make_uint4(0u, 0u, 0u, 0u);
}

// D = rowsum(dO * O) and l2 = LSE * log2(e) (+inf for a row without any visible key, so
// that 2^(x - l2) = 0) for every query row; one warp per row.
__global__ void attn_bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ o,
                                       const __nv_bfloat16* __restrict__ dout,
                                       const float* __restrict__ lse, float* dvec, float* l2,
                                       long long rows, int Dh) {
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(o + row * Dh);
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(dout + row * Dh);
  float acc = 0.f;
  for (int c = lane; c < Dh / 2; c += 32) {
    const float2 x = __bfloat1622float2(a[c]);
    const float2 y = __bfloat1622float2(b[c]);
    acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    dvec[row] = acc;
    const float L = lse[row];
    l2[row] = (L == -INFINITY) ? INFINITY : L * kLog2eB;
  }
}

// Shared pieces of the two gradient kernels: the barrier layout and the tcgen05 issue of
// one streamed tile pair (two SS products into X and Y, then TS products from X / Y).
template <int D>
struct BwdSmem {
  uint32_t stat, ring, bars;
  uint8_t* base;
  __device__ __forceinline__ uint32_t bar(int i) const { return bars + 8u * (uint32_t)i; }
};

template <int D>
__device__ __forceinline__ BwdSmem<D> bwd_smem(uint8_t* smem_raw) {
  using C = BwdCfg<D>;
  BwdSmem<D> s;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  s.base = smem_raw + (base - raw);
  s.stat = base + C::kStatOff;
  s.ring = base + C::kRingOff;
  s.bars = base + C::kBarOff;
  return s;
}

// X or Y = A_stat[a] (stationary tile a, K-major) times B^T (ring tile, K-major): 128 x 128.
template <int D>
__device__ __forceinline__ void issue_ss(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
  using C = BwdCfg<D>;
  constexpr uint32_t idesc = idesc_bf16_f32(kBT, kBT, false);
  const uint64_t da = smem_desc(a_smem, 16, 1024);
  const uint64_t db = smem_desc(b_smem, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * C::kChunkBytes + (kk & 3) * 32) >> 4;
    umma_ss_warp(d_tmem, da + off, db + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// acc (128 x D) += A (bf16 pairs in TMEM: contraction step kk at column 8 kk, plus 32 for
// kk >= 4, the second warpgroup's half) times B (ring tile: 128 rows along the contraction,
// D columns, MN-major).
template <int D>
__device__ __forceinline__ void issue_ts(uint32_t acc, uint32_t a_tmem, uint32_t b_smem,
                                         bool first) {
  using C = BwdCfg<D>;
  constexpr uint32_t idesc = idesc_bf16_f32(kBT, D, true);
  const uint64_t db = smem_desc(b_smem, C::kChunkBytes, 1024);
#pragma unroll
  for (int kk = 0; kk < kBT / 16; ++kk)
    umma_ts_warp(acc, a_tmem + 8u * kk + (kk >= 4 ? 32u : 0u), db + ((kk * 16 * 128) >> 4),
                 idesc, (!first || kk > 0) ? 1u : 0u);
}

// dQ of one 128-row query tile of head (b, h).  kAlibi: the scores carry the ALiBi bias
// -slope_h |q - kv|, which moves each P element's base-2 offset from l2 to l2 + slope2 |q - kv|.
template <int D, bool kAlibi, bool kCap>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const BwdParams p) {
  using C = DqCfg<D>;
  using CB = BwdCfg<D>;
  constexpr int SK = C::kSlotsK, SV = C::kSlotsV;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);
  const uint32_t sStat = base_u32 + C::kStatOff;
  auto k_tile = [&](int t) { return base_u32 + C::kKOff + (uint32_t)(t % SK) * C::kTileBytes; };
  auto v_tile = [&](int t) { return base_u32 + C::kVOff + (uint32_t)(t % SV) * C::kTileBytes; };
  auto bar = [&](int i) { return base_u32 + C::kBarOff + 8u * (uint32_t)i; };
  // S ready, dP ready, X free (S loaded into registers), dS ready
  const int BAR_STAT = 0, BAR_S = C::kOwn, BAR_DP = C::kOwn + 1, BAR_XF = C::kOwn + 2,
            BAR_DS = C::kOwn + 3, BAR_ACC = C::kOwn + 4, BAR_DONE = C::kOwn + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::kBarOff + C::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int nqt = (p.Nq + kBT - 1) / kBT;
  const int bh = blockIdx.x / nqt, qt = blockIdx.x % nqt;
  const int b = bh / p.Hq, h = bh % p.Hq, hk = h / p.G;
  const int q0 = qt * kBT;
  int lo_first, hi_first, lo_last, hi_last;
  row_interval(p.mask, q0, lo_first, hi_first);
  row_interval(p.mask, min(q0 + kBT, p.Nq) - 1, lo_last, hi_last);
  int ja = 0, n = 0;                    // K/V tiles [ja, ja + n) that the tile's rows see
  if (p.Nk > 0 && hi_last >= lo_first) {
    ja = lo_first / kBT;
    n = hi_last / kBT - ja + 1;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kOwn; ++i) mbar_init(bar(i), 1);   // stat, both rings
    mbar_init(bar(BAR_S), 1);
    mbar_init(bar(BAR_DP), 1);
    mbar_init(bar(BAR_XF), 8);
    mbar_init(bar(BAR_DS), 8);
    mbar_init(bar(BAR_ACC), 1);
    mbar_init(bar(BAR_DONE), 1);
    *abort_flag = 0;
    init_wait_limit(abort_flag, p.err);
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kBwdMmaWarp) {
   regs_decrease<kBwdRegsOther>();
   if (warp == kBwdTmaWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n > 0) {
      mbar_arrive_expect_tx(bar(BAR_STAT), 2 * C::kTileBytes);
#pragma unroll
      for (int c = 0; c < CB::kChunks; ++c) {
        tma_load_3d(sStat + c * CB::kChunkBytes, &tmQ, bar(BAR_STAT), c * 64, q0, bh);
        tma_load_3d(sStat + C::kTileBytes + c * CB::kChunkBytes, &tmDO, bar(BAR_STAT), c * 64,
                    q0, bh);
      }
      const int zkv = b * p.Hkv + hk;
      int tk = 0, tv = 0;                    // tiles issued into the K and V rings
      for (int t = 0; t < n; ++t) {
        const int row = (ja + t) * kBT;
        if (t >= SK && !mbar_wait(bar(C::kEmptyK + t % SK), (t / SK - 1) & 1, abort_flag, p.err,
                                  kSiteBwdEmpty))
          break;
        mbar_arrive_expect_tx(bar(C::kFullK + t % SK), C::kTileBytes);
#pragma unroll
        for (int c = 0; c < CB::kChunks; ++c)
          tma_load_3d(k_tile(t) + c * CB::kChunkBytes, &tmK, bar(C::kFullK + t % SK), c * 64,
                      row, zkv);
        ++tk;
        if (t >= SV && !mbar_wait(bar(C::kEmptyV + t % SV), (t / SV - 1) & 1, abort_flag, p.err,
                                  kSiteBwdEmpty))
          break;
        mbar_arrive_expect_tx(bar(C::kFullV + t % SV), C::kTileBytes);
#pragma unroll
        for (int c = 0; c < CB::kChunks; ++c)
          tma_load_3d(v_tile(t) + c * CB::kChunkBytes, &tmV, bar(C::kFullV + t % SV), c * 64,
                      row, zkv);
        ++tv;
      }
      // outstanding copies land before the CTA may exit (matters only on abort)
      mbar_wait(bar(BAR_STAT), 0, nullptr, p.err, kSiteBwdDrain);
      for (int s = 0; s < SK && s < tk; ++s) {
        const int last = s + ((tk - 1 - s) / SK) * SK;
        mbar_wait(bar(C::kFullK + s), (last / SK) & 1, nullptr, p.err, kSiteBwdDrain);
      }
      for (int s = 0; s < SV && s < tv; ++s) {
        const int last = s + ((tv - 1 - s) / SV) * SV;
        mbar_wait(bar(C::kFullV + s), (last / SV) & 1, nullptr, p.err, kSiteBwdDrain);
      }
    }
    __syncwarp();
   } else if (warp == kBwdMmaWarp) {
    // -------------------------------------------------------------- tcgen05 issuer
    if (n > 0) {
      bool ok = mbar_wait_warp(bar(BAR_STAT), 0, abort_flag, p.err, kSiteBwdStat);
      tc_fence_after();
      // Order: S_0, dP_0, then per tile t: S_{t+1} as soon as the element-wise groups hold
      // S_t in registers, dQ += dS_t K_t once dS_t is written, dP_{t+1} behind it (dP_{t+1}
      // overwrites Y, which dQ reads first: the tensor pipe runs in order).  The products of
      // the next tile overlap the element-wise work of this one.  A K tile is released after
      // its dQ product, a V tile after its dP product.
      auto full_k = [&](int t) {
        const bool f = mbar_wait_warp(bar(C::kFullK + t % SK), (t / SK) & 1, abort_flag, p.err,
                                      kSiteBwdFull);
        tc_fence_after();
        return f;
      };
      auto full_v = [&](int t) {
        const bool f = mbar_wait_warp(bar(C::kFullV + t % SV), (t / SV) & 1, abort_flag, p.err,
                                      kSiteBwdFull);
        tc_fence_after();
        return f;
      };
      if (ok && full_k(0) && full_v(0)) {
        issue_ss<D>(tmem + kTmemX, sStat, k_tile(0));                               // S_0
        umma_commit_warp(bar(BAR_S));
        issue_ss<D>(tmem + kTmemY, sStat + C::kTileBytes, v_tile(0));               // dP_0
        umma_commit_warp(bar(BAR_DP));
        umma_commit_warp(bar(C::kEmptyV + 0));
      } else {
        ok = false;
      }
      for (int t = 0; ok && t < n; ++t) {
        if (t + 1 < n) {
          if (!mbar_wait_warp(bar(BAR_XF), t & 1, abort_flag, p.err, kSiteBwdP) || !full_k(t + 1))
            break;
          issue_ss<D>(tmem + kTmemX, sStat, k_tile(t + 1));                       // S_{t+1}
          umma_commit_warp(bar(BAR_S));
        }
        if (!mbar_wait_warp(bar(BAR_DS), t & 1, abort_flag, p.err, kSiteBwdP)) break;
        tc_fence_after();
        issue_ts<D>(tmem + kTmemAcc0, tmem + kTmemY, k_tile(t), t == 0);     // dQ += dS K
        umma_commit_warp(bar(C::kEmptyK + t % SK));
        if (t + 1 < n) {
          if (!full_v(t + 1)) break;
          issue_ss<D>(tmem + kTmemY, sStat + C::kTileBytes, v_tile(t + 1));
          umma_commit_warp(bar(BAR_DP));                                       // dP_{t+1}
          umma_commit_warp(bar(C::kEmptyV + (t + 1) % SV));
        }
      }
      umma_commit_warp(bar(BAR_ACC));
    }
    umma_commit_warp(bar(BAR_DONE));
    mbar_wait_warp(bar(BAR_DONE), 0, nullptr, p.err, kSiteBwdDrain);
   }
  } else {
    regs_increase<kBwdRegsElem>();
    // ----------------------------------------------------- element-wise warpgroups
    const int g = warp >> 2;                   // key columns [64g, 64g + 64) of each tile
    const int wq = warp & 3;                   // TMEM lane quarter
    const int r = wq * 32 + lane;
    const int row = q0 + r;
    const bool valid = row < p.Nq;
    const long long ridx = (long long)bh * p.Nq + row;
    const float l2r = valid ? p.l2[ridx] : INFINITY;
    const float dr = valid ? p.dvec[ridx] : 0.f;
    const float4 l2r4 = make_float4(l2r, l2r, l2r, l2r);
    const float4 dr4 = make_float4(dr, dr, dr, dr);
    const float slope2 = kAlibi ? __ldg(p.alibi + h) * kLog2eB : 0.f;
    const float inv_cap = kCap ? 1.f / p.cap_log2 : 0.f;
    int rlo = 1, rhi = 0;
    if (valid) row_interval(p.mask, row, rlo, rhi);
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t col = 64u * (uint32_t)g;
    __nv_bfloat16* drow = reinterpret_cast<__nv_bfloat16*>(p.dq) + ridx * D;
    bool ok = true;
    for (int t = 0; ok && t < n; ++t) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_S), t & 1, abort_flag, p.err, kSiteBwdS));
      if (!ok) break;
      tc_fence_after();
      const int k0 = (ja + t) * kBT;
      const bool full = lo_last <= k0 && k0 + kBT - 1 <= hi_first && k0 + kBT <= p.Nk;
      const int kc = k0 + (int)col;
      auto vis = [&](int c) -> unsigned {      // columns kc + c .. kc + c + 3
        if (full) return 0xFu;
        unsigned m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) m |= (kc + c + i >= rlo && kc + c + i <= rhi) ? (1u << i) : 0u;
        return m;
      };
      uint32_t s[64];
      tmem_ld_x64_async(tl + kTmemX + col, s);
      tmem_ld_wait_x64(s);
      // S_t is in registers: X may take S_{t+1}
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_XF));
      if constexpr (kAlibi) {
        // key kc + c is |row - kc - c| away from this row
        const float drow = (float)(row - kc);
        probs<64>(s, p.kscale, [&](int j) {
          const float c = (float)(4 * j);
          return make_float4(fmaf(slope2, fabsf(drow - c), l2r), fmaf(slope2, fabsf(drow - c - 1.f), l2r),
                             fmaf(slope2, fabsf(drow - c - 2.f), l2r), fmaf(slope2, fabsf(drow - c - 3.f), l2r));
        }, [&](int j) { return vis(4 * j); }, p);
      } else {
        // with the cap, s keeps the exponents: nothing reads P before the grads step
        probs<64, kCap, kCap>(s, p.kscale, [&](int) { return l2r4; },
                              [&](int j) { return vis(4 * j); }, p);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_DP), t & 1, abort_flag, p.err, kSiteBwdS));
      if (!ok) break;
      tc_fence_after();
      uint32_t dp[64];
      tmem_ld_x64_async(tl + kTmemY + col, dp);
      tmem_ld_wait_x64(dp);
      {
        uint32_t pk[16], dsk[16];
        grads<false, 0, 64, 64, kCap, kCap>(s, dp, [&](int) { return dr4; }, pk, dsk,
                                            [&](int) { return l2r4; }, inv_cap);
        tmem_st_x16(tl + kTmemY + col, dsk);
      }
      {
        uint32_t pk[16], dsk[16];
        grads<false, 32, 64, 64, kCap, kCap>(s, dp, [&](int) { return dr4; }, pk, dsk,
                                             [&](int) { return l2r4; }, inv_cap);
        tmem_st_x16(tl + kTmemY + col + 16u, dsk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_DS));
    }
    // group g writes dQ columns [g D / 2, (g + 1) D / 2) of its row
    if (n == 0) {
      store_zero_row(drow + g * (D / 2), D / 2, valid);
    } else if (ok) {
      const bool okacc =
          __all_sync(0xffffffffu, mbar_wait(bar(BAR_ACC), 0, abort_flag, p.err, kSiteBwdAcc));
      if (okacc) {
        tc_fence_after();
        store_row<D / 2>(tl + kTmemAcc0 + (uint32_t)(g * (D / 2)), p.scale, drow + g * (D / 2),
                         valid);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// dK and dV of one 128-key tile of KV head (b, hk), summed over the query heads of its group
// (kAlibi as for attn_bwd_dq_kernel, with the slope of each streamed tile's query head).
template <int D, bool kAlibi, bool kCap>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const BwdSmem<D> sm = bwd_smem<D>(smem_raw);
  // S^T ready, dP^T ready, P^T written, dS^T written
  const int BAR_STAT = 0, BAR_FULL = 1, BAR_EMPTY = 1 + NS, BAR_S = 1 + 2 * NS,
            BAR_DP = 2 + 2 * NS, BAR_P = 3 + 2 * NS, BAR_DS = 4 + 2 * NS,
            BAR_ACC = 5 + 2 * NS, BAR_DONE = 6 + 2 * NS, BAR_VF = 7 + 2 * NS,
            BAR_VE = 9 + 2 * NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm.base + C::kBarOff + C::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // per streamed query tile: base-2 LSE, D, and each query's visible key interval
  float* vec = reinterpret_cast<float*>(sm.base + C::kVecOff);     // [2][4][128]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int nkt = (p.Nk + kBT - 1) / kBT;
  const int bk = blockIdx.x / nkt, kt = blockIdx.x % nkt;
  const int b = bk / p.Hkv, hk = bk % p.Hkv;
  const int k0 = kt * kBT;
  const int k1 = min(k0 + kBT, p.Nk) - 1;
  int qa, qb;
  query_range(p.mask, p.Nq, k0, k1, qa, qb);
  int ia = 0, ni = 0;                 // query tiles [ia, ia + ni) of every head of the group
  if (qa <= qb) {
    ia = qa / kBT;
    ni = qb / kBT - ia + 1;
  }
  const int n = ni * p.G;             // streamed tiles: head g of the group, query tile i

  if (threadIdx.x == 0) {
    mbar_init(sm.bar(BAR_STAT), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(sm.bar(BAR_FULL + s), 1);
      mbar_init(sm.bar(BAR_EMPTY + s), 1);
    }
    mbar_init(sm.bar(BAR_S), 1);
    mbar_init(sm.bar(BAR_DP), 1);
    mbar_init(sm.bar(BAR_P), 8);
    mbar_init(sm.bar(BAR_DS), 8);
    mbar_init(sm.bar(BAR_ACC), 1);
    mbar_init(sm.bar(BAR_DONE), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.bar(BAR_VF + i), 64);     // every thread of warps 10-11
      mbar_init(sm.bar(BAR_VE + i), 8);      // every element-wise warp
    }
    *abort_flag = 0;
    init_wait_limit(abort_flag, p.err);
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kBwdMmaWarp) {
   regs_decrease<kBwdRegsOther>();
   if (warp > kBwdTmaWarp) {
    // ------------------------------------------------- per-query vectors of each tile
    // l2 = LSE log2(e), D and the visible key interval of the tile's 128 queries, into the
    // parity buffer of the tile, ahead of the element-wise groups.
    const int i = (warp - kBwdTmaWarp - 1) * 32 + lane;     // 0..63
    for (int t = 0; t < n; ++t) {
      const int par = t & 1;
      if (t >= 2 && !mbar_wait(sm.bar(BAR_VE + par), ((t >> 1) - 1) & 1, abort_flag, p.err,
                               kSiteBwdVecEmpty))
        break;
      const int h = hk * p.G + t / ni;
      const int q0 = (ia + t % ni) * kBT;
#pragma unroll
      for (int e = i; e < kBT; e += 64) {
        const int q = q0 + e;
        float l2q = INFINITY, dq = 0.f;
        int lo = 1, hi = 0;
        if (q < p.Nq) {
          const long long qi = ((long long)b * p.Hq + h) * p.Nq + q;
          l2q = p.l2[qi];
          dq = p.dvec[qi];
          row_interval(p.mask, q, lo, hi);
        }
        vec[(par * 4 + 0) * kBT + e] = l2q;
        vec[(par * 4 + 1) * kBT + e] = dq;
        vec[(par * 4 + 2) * kBT + e] = __int_as_float(lo);
        vec[(par * 4 + 3) * kBT + e] = __int_as_float(hi);
      }
      mbar_arrive(sm.bar(BAR_VF + par));
    }
   } else if (warp == kBwdTmaWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n > 0) {
      const int zkv = b * p.Hkv + hk;
      mbar_arrive_expect_tx(sm.bar(BAR_STAT), 2 * C::kTileBytes);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c) {
        tma_load_3d(sm.stat + c * C::kChunkBytes, &tmK, sm.bar(BAR_STAT), c * 64, k0, zkv);
        tma_load_3d(sm.stat + C::kTileBytes + c * C::kChunkBytes, &tmV, sm.bar(BAR_STAT),
                    c * 64, k0, zkv);
      }
      int t = 0;
      for (; t < n; ++t) {
        const int s = t % NS, round = t / NS;
        if (round > 0 &&
            !mbar_wait(sm.bar(BAR_EMPTY + s), (round - 1) & 1, abort_flag, p.err, kSiteBwdEmpty))
          break;
        const int h = hk * p.G + t / ni;
        const int row = (ia + t % ni) * kBT;
        const int zq = b * p.Hq + h;
        mbar_arrive_expect_tx(sm.bar(BAR_FULL + s), 2 * C::kTileBytes);
        const uint32_t dst = sm.ring + s * 2 * C::kTileBytes;
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_3d(dst + c * C::kChunkBytes, &tmQ, sm.bar(BAR_FULL + s), c * 64, row, zq);
          tma_load_3d(dst + C::kTileBytes + c * C::kChunkBytes, &tmDO, sm.bar(BAR_FULL + s),
                      c * 64, row, zq);
        }
      }
      mbar_wait(sm.bar(BAR_STAT), 0, nullptr, p.err, kSiteBwdDrain);
      for (int s = 0; s < NS && s < t; ++s) {
        const int last = s + ((t - 1 - s) / NS) * NS;
        mbar_wait(sm.bar(BAR_FULL + s), (last / NS) & 1, nullptr, p.err, kSiteBwdDrain);
      }
    }
    __syncwarp();
   } else if (warp == kBwdMmaWarp) {
    // -------------------------------------------------------------- tcgen05 issuer
    if (n > 0) {
      bool ok = mbar_wait_warp(sm.bar(BAR_STAT), 0, abort_flag, p.err, kSiteBwdStat);
      tc_fence_after();
      // Order: S^T_0, dP^T_0, then per tile t: dV += P^T_t dO_t once P^T_t is written,
      // S^T_{t+1} behind it (it overwrites X, which dV reads first: the tensor pipe runs in
      // order), dK += dS^T_t Q_t once dS^T_t is written, dP^T_{t+1} behind it.  Each pair of
      // products overlaps one of the two element-wise steps.
      auto stage = [&](int t) { return sm.ring + (t % NS) * 2 * C::kTileBytes; };
      auto full = [&](int t) {
        const bool f = mbar_wait_warp(sm.bar(BAR_FULL + t % NS), (t / NS) & 1, abort_flag,
                                      p.err, kSiteBwdFull);
        tc_fence_after();
        return f;
      };
      if (ok && full(0)) {
        issue_ss<D>(tmem + kTmemX, sm.stat, stage(0));                              // S^T_0
        umma_commit_warp(sm.bar(BAR_S));
        issue_ss<D>(tmem + kTmemY, sm.stat + C::kTileBytes, stage(0) + C::kTileBytes);  // dP^T_0
        umma_commit_warp(sm.bar(BAR_DP));
      } else {
        ok = false;
      }
      for (int t = 0; ok && t < n; ++t) {
        const uint32_t qt = stage(t);
        if (!mbar_wait_warp(sm.bar(BAR_P), t & 1, abort_flag, p.err, kSiteBwdP)) break;
        tc_fence_after();
        issue_ts<D>(tmem + kTmemAcc0, tmem + kTmemX, qt + C::kTileBytes, t == 0);  // dV
        if (t + 1 < n) {
          if (!full(t + 1)) break;
          issue_ss<D>(tmem + kTmemX, sm.stat, stage(t + 1));                      // S^T_{t+1}
          umma_commit_warp(sm.bar(BAR_S));
        }
        if (!mbar_wait_warp(sm.bar(BAR_DS), t & 1, abort_flag, p.err, kSiteBwdP)) break;
        tc_fence_after();
        issue_ts<D>(tmem + kTmemAcc1, tmem + kTmemY, qt, t == 0);                 // dK
        umma_commit_warp(sm.bar(BAR_EMPTY + t % NS));
        if (t + 1 < n) {
          issue_ss<D>(tmem + kTmemY, sm.stat + C::kTileBytes, stage(t + 1) + C::kTileBytes);
          umma_commit_warp(sm.bar(BAR_DP));                                    // dP^T_{t+1}
        }
      }
      umma_commit_warp(sm.bar(BAR_ACC));
    }
    umma_commit_warp(sm.bar(BAR_DONE));
    mbar_wait_warp(sm.bar(BAR_DONE), 0, nullptr, p.err, kSiteBwdDrain);
   }
  } else {
    regs_increase<kBwdRegsElem>();
    // ----------------------------------------------------- element-wise warpgroups
    const int g = warp >> 2;         // query columns [64g, 64g + 64) of each streamed tile
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const int key = k0 + r;
    const bool kvalid = key < p.Nk;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t col = 64u * (uint32_t)g;
    const long long kidx = ((long long)b * p.Hkv + hk) * p.Nk + key;
    const float inv_cap = kCap ? 1.f / p.cap_log2 : 0.f;
    bool ok = true;
    for (int t = 0; t < n; ++t) {
      // this tile's query vectors, written ahead by warps 10-11
      const int par = t & 1;
      const int q0 = (ia + t % ni) * kBT;
      ok = __all_sync(0xffffffffu, mbar_wait(sm.bar(BAR_VF + par), (t >> 1) & 1, abort_flag,
                                             p.err, kSiteBwdVecFull));
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(sm.bar(BAR_S), t & 1, abort_flag, p.err, kSiteBwdS));
      if (!ok) break;
      tc_fence_after();
      const float* l2v = vec + (par * 4 + 0) * kBT + col;
      const float* dv = vec + (par * 4 + 1) * kBT + col;
      const int* lov = reinterpret_cast<const int*>(vec + (par * 4 + 2) * kBT + col);
      const int* hiv = reinterpret_cast<const int*>(vec + (par * 4 + 3) * kBT + col);
      // Every query of the group's 64 sees every key of the CTA's tile (the intervals are
      // non-decreasing at both ends, so the last query's start and the first query's end
      // decide): no per-pair test.
      const bool full = q0 + (int)col + 64 <= p.Nq && k0 + kBT <= p.Nk && lov[63] <= k0 &&
                        k1 <= hiv[0];
      auto vis = [&](int c) -> unsigned {      // group columns c .. c + 3
        if (full) return 0xFu;
        const int4 lo = *reinterpret_cast<const int4*>(lov + c);
        const int4 hi = *reinterpret_cast<const int4*>(hiv + c);
        unsigned m = 0;
        if (kvalid) {
          m |= (lo.x <= key && key <= hi.x) ? 1u : 0u;
          m |= (lo.y <= key && key <= hi.y) ? 2u : 0u;
          m |= (lo.z <= key && key <= hi.z) ? 4u : 0u;
          m |= (lo.w <= key && key <= hi.w) ? 8u : 0u;
        }
        return m;
      };
      // ALiBi: query q0 + col + c is |key - q0 - col - c| away from this key
      const float slope2 = kAlibi ? __ldg(p.alibi + hk * p.G + t / ni) * kLog2eB : 0.f;
      const float dkey = (float)(key - q0 - (int)col);
      auto l2f = [&](int c) {
        float4 l = *reinterpret_cast<const float4*>(l2v + c);
        if constexpr (kAlibi) {
          const float fc = (float)c;
          l.x = fmaf(slope2, fabsf(dkey - fc), l.x);
          l.y = fmaf(slope2, fabsf(dkey - fc - 1.f), l.y);
          l.z = fmaf(slope2, fabsf(dkey - fc - 2.f), l.z);
          l.w = fmaf(slope2, fabsf(dkey - fc - 3.f), l.w);
        }
        return l;
      };
      auto dvf = [&](int c) { return *reinterpret_cast<const float4*>(dv + c); };
      // Step 1 (S^T ready): P^T of the group's 64 columns, in two halves of 32; the bf16
      // P^T of a half lands in columns the group has already read.
      uint32_t pr0[32], pr1[32];
      {
        uint32_t pk[16];
        tmem_ld_x32_async(tl + kTmemX + col, pr0);
        tmem_ld_wait_x32(pr0);
        probs<32, kCap>(pr0, p.kscale, [&](int j) { return l2f(4 * j); },
                        [&](int j) { return vis(4 * j); }, p);
        pack_pairs(pr0, pk);
        tmem_st_x16(tl + kTmemX + col, pk);
        tmem_ld_x32_async(tl + kTmemX + col + 32u, pr1);
        tmem_ld_wait_x32(pr1);
        probs<32, kCap>(pr1, p.kscale, [&](int j) { return l2f(32 + 4 * j); },
                        [&](int j) { return vis(32 + 4 * j); }, p);
        pack_pairs(pr1, pk);
        tmem_st_x16(tl + kTmemX + col + 16u, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.bar(BAR_P));
      // Step 2 (dP^T ready): dS^T = P^T (dP^T - D), into the low half of Y likewise.
      ok = __all_sync(0xffffffffu, mbar_wait(sm.bar(BAR_DP), t & 1, abort_flag, p.err, kSiteBwdS));
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t dph[32], pk[16], dsk[16];
        tmem_ld_x32_async(tl + kTmemY + col, dph);
        tmem_ld_wait_x32(dph);
        grads<false, 0, 32, 32, kCap>(pr0, dph, [&](int j) { return dvf(4 * j); }, pk, dsk,
                                      [&](int j) { return l2f(4 * j); }, inv_cap);
        tmem_st_x16(tl + kTmemY + col, dsk);
        tmem_ld_x32_async(tl + kTmemY + col + 32u, dph);
        tmem_ld_wait_x32(dph);
        grads<false, 0, 32, 32, kCap>(pr1, dph, [&](int j) { return dvf(32 + 4 * j); }, pk, dsk,
                                      [&](int j) { return l2f(32 + 4 * j); }, inv_cap);
        tmem_st_x16(tl + kTmemY + col + 16u, dsk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sm.bar(BAR_DS));
        mbar_arrive(sm.bar(BAR_VE + par));    // this warp has read the tile's vectors
      }
    }
    // group 0 writes the dV row, group 1 the dK row
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(g == 0 ? p.dv : p.dk) + kidx * D;
    if (n == 0) {
      store_zero_row(dst, D, kvalid);
    } else if (ok) {
      const bool okacc =
          __all_sync(0xffffffffu, mbar_wait(sm.bar(BAR_ACC), 0, abort_flag, p.err, kSiteBwdAcc));
      if (okacc) {
        tc_fence_after();
        if (g == 0)
          store_row<D>(tl + kTmemAcc0, 1.f, dst, kvalid);
        else
          store_row<D>(tl + kTmemAcc1, p.scale, dst, kvalid);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool kAlibi, bool kCap>
int launch_bwd_t(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                 const CUtensorMap& tv, const BwdParams& p, cudaStream_t stream) {
  using C = BwdCfg<D>;
  using CQ = DqCfg<D>;
  static_assert(C::kSmemBytes <= 227 * 1024 && CQ::kSmemBytes <= 227 * 1024,
                "shared memory budget");
  if (cudaFuncSetAttribute(attn_bwd_dq_kernel<D, kAlibi, kCap>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           CQ::kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D, kAlibi, kCap>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes) != cudaSuccess)
    return -4;
  const long long nq = (long long)p.B * p.Hq * ((p.Nq + kBT - 1) / kBT);
  const long long nk = (long long)p.B * p.Hkv * ((p.Nk + kBT - 1) / kBT);
  if (nk > 0)
    attn_bwd_dkdv_kernel<D, kAlibi, kCap><<<(unsigned)nk, kBwdThreads, C::kSmemBytes, stream>>>(tq, tdo, tk,
                                                                                 tv, p);
  if (nq > 0)
    attn_bwd_dq_kernel<D, kAlibi, kCap><<<(unsigned)nq, kBwdThreads, CQ::kSmemBytes, stream>>>(tq, tdo, tk,
                                                                                tv, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace

int launch_bwd_rowdot(const void* o, const void* dout, const float* lse, float* dvec, float* l2,
                      long long rows, int d, cudaStream_t stream) {
  if (rows <= 0) return 0;
  const int warps = 8;
  const long long blocks = (rows + warps - 1) / warps;
  attn_bwd_rowdot_kernel<<<(unsigned)blocks, warps * 32, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(o), reinterpret_cast<const __nv_bfloat16*>(dout),
      lse, dvec, l2, rows, d);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

int launch_attn_bwd(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                    const CUtensorMap& tv, const BwdParams& p, int d, cudaStream_t stream) {
  // ALiBi and the soft-cap are not combined (the host refuses that request)
  const bool alibi = p.alibi != nullptr, cap = p.cap_scale > 0.f;
  if (alibi && cap) return -2;
  if (d == 128) return alibi ? launch_bwd_t<128, true, false>(tq, tdo, tk, tv, p, stream)
                       : cap ? launch_bwd_t<128, false, true>(tq, tdo, tk, tv, p, stream)
                             : launch_bwd_t<128, false, false>(tq, tdo, tk, tv, p, stream);
  if (d == 64) return alibi ? launch_bwd_t<64, true, false>(tq, tdo, tk, tv, p, stream)
                      : cap ? launch_bwd_t<64, false, true>(tq, tdo, tk, tv, p, stream)
                            : launch_bwd_t<64, false, false>(tq, tdo, tk, tv, p, stream);
  return -2;
}

}  // namespace attn
