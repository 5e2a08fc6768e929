// Fused exact attention forward for sm_100a: O = softmax(scale * Q K^T + mask) V and the
// row log-sum-exp, in one pass; S and P never leave the SM.
//
// The algorithm is the tiled online softmax of "FlashAttention 논문 분석: IO-Aware Exact
// Attention" (sections "Online Softmax와 블록 단위 누적" and "알고리즘 의사코드"): for each
// K/V tile the running row max m and exp-sum l are updated and the output is rescaled, so
// each row's softmax is exact even though no tile sees the whole row ("Attention 최적화가
// 어려운 이유", section "나머지 점수가 바꾸는 확률").  The FlashAttention-2/3 refinements the
// same page lists -- one final normalisation instead of one per tile, mask math only on
// tiles that need it, the grid over query blocks, producer/consumer warp specialisation,
// TMA loads and the GEMM/softmax overlap between two query tiles -- are re-expressed for
// Blackwell:
//
//   * a persistent grid (one CTA per SM) walks query pairs: two 128-row query tiles
//     (t = 0, 1) of one (batch, head); the K/V tiles they need stream through a TMA ring in
//     shared memory (128B-swizzled) that never drains between pairs; each query tile only
//     visits the K/V tiles its own rows can see;
//   * warp 8 issues tcgen05.mma: S_t = Q_t K_j^T into TMEM columns [128t, 128t+128), then
//     O_t += P_t V_j with P_t read straight from TMEM columns [128t+64, 128t+128) and O_t
//     accumulated in TMEM columns [256+128t, ...);
//   * warp 9 issues the K/V TMA loads, warp 10 reloads each query tile's Q as soon as its
//     last QK^T of the previous pair is done (warp 11 is spare);
//   * warps 0-3 and 4-7 are the softmax warpgroups of tile 0 and tile 1: thread r owns row
//     r of its tile, reads its 128 scores from TMEM, applies mask / scale / soft-cap,
//     updates (m, l), rescales its O row in TMEM only when the running max has grown by
//     more than 2^8 (exact: the final division uses the same reference max), and writes
//     P back to TMEM as bf16;
//   * the two softmax warpgroups ping-pong: while one computes exponentials, the tensor
//     core runs the other tile's MMAs.
// The epilogue divides O by l, rounds to bf16 and writes LSE = (m + log2 l) * ln 2.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "attn_internal.h"
#include "mask.cuh"
#include "sm100_ptx.cuh"
#include "tmem_ldst.cuh"

namespace attn {

namespace {

constexpr int kBM = 128;               // rows per query tile (TMEM lanes)
constexpr int kBN = 128;               // keys per K/V tile
constexpr int kThreads = 384;          // 2 softmax warpgroups + {MMA, K/V TMA, Q TMA, spare}
constexpr int kMmaWarp = 8;
constexpr int kTmaWarp = 9;
constexpr int kQWarp = 10;
// Registers per thread after the split; the launch gives 168 (65536 / 384, rounded down to
// a multiple of 8): 2 * 128 * 192 + 128 * 112 = 63488 <= 384 * 168 = 64512.  The soft-cap
// variant holds its polynomial's coefficients beside the row and takes
// 2 * 128 * 200 + 128 * 104 = 64512.
constexpr uint32_t kRegsSoftmax = 192;
constexpr uint32_t kRegsOther = 112;
constexpr uint32_t kRegsSoftmaxCap = 200;
constexpr uint32_t kRegsOtherCap = 104;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale when max grows > 2^8
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kLog2eF = 1.44269504088896341f;
constexpr uint32_t kNegInfBits = 0xff800000u;

template <int D, bool kFp8 = false>
struct Cfg {
  static constexpr int kElem = kFp8 ? 1 : 2;        // bytes per element (E4M3 or bf16)
  static constexpr int kChunks = D * kElem / 128;   // 128-byte swizzle atoms along d
  static constexpr int kChunkBytes = kBM * 128;     // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBM * D * kElem;  // one Q, K or V tile
  static constexpr int kStages = (kTileBytes >= 32768) ? 4 : 8;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
  // barriers: q[2], q_free[2], full[S], empty[S], s[2], p[2][2 key halves], o[2], done
  static constexpr int kNumBars = 13 + 2 * kStages;
  // after the barriers: TMEM slot, abort flag and wait limit (16 bytes), then this CTA's
  // work list when the grid is scheduled by cost (count + up to kSchedMax unit indices)
  static constexpr int kSchedOff = kBarOff + kNumBars * 8 + 16;
  static constexpr int kSmemBytes = kSchedOff + 4 * (1 + kSchedMax) + 1024;
};

enum : uint32_t {
  kSiteQ = 1, kSiteEmpty, kSiteFullK, kSiteFullV, kSitePFull, kSiteSFull, kSiteOFinal,
  kSiteDrain, kSiteQFree,
};

__device__ __forceinline__ float f32(uint32_t u) { return __uint_as_float(u); }

// Row maximum of the raw scores of one tile row.  Masked columns (outside [c_lo, c_hi])
// are overwritten with -inf first.  The scale is positive and the soft-cap is increasing,
// so the maximum of the transformed scores is the transform of this maximum.  Four
// independent chains of 3-input maxima keep the dependency depth at 16.
template <bool kMasked>
__device__ __forceinline__ float tile_row_max(uint32_t (&s)[128], int c_lo, int c_hi) {
  if (kMasked) {
#pragma unroll
    for (int c = 0; c < 128; ++c)
      if ((unsigned)(c - c_lo) > (unsigned)(c_hi - c_lo)) s[c] = kNegInfBits;
  }
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
  for (int c = 0; c < 128; c += 8) {
    m0 = max3f(m0, f32(s[c]), f32(s[c + 1]));
    m1 = max3f(m1, f32(s[c + 2]), f32(s[c + 3]));
    m2 = max3f(m2, f32(s[c + 4]), f32(s[c + 5]));
    m3 = max3f(m3, f32(s[c + 6]), f32(s[c + 7]));
  }
  return max3f(m0, m1, fmaxf(m2, m3));
}

// Largest |s| of a tile row (all 128 columns; masked ones included, which only makes the
// soft-cap path's range test stricter).
__device__ __forceinline__ float tile_row_absmax(const uint32_t (&s)[128]) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int c = 0; c < 128; c += 8) {
    a0 = max3f(a0, fabsf(f32(s[c])), fabsf(f32(s[c + 1])));
    a1 = max3f(a1, fabsf(f32(s[c + 2])), fabsf(f32(s[c + 3])));
    a2 = max3f(a2, fabsf(f32(s[c + 4])), fabsf(f32(s[c + 5])));
    a3 = max3f(a3, fabsf(f32(s[c + 6])), fabsf(f32(s[c + 7])));
  }
  return fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
}

// The soft-cap polynomial of p.cap_poly at one raw score s (|s| <= cap_fast_max): the
// base-2 capped score c log2(e) tanh(s scale / c) = s (b0 + w (b1 + w (b2 + w (b3 + w b4)))),
// w = s^2, c log2(e) and the powers of scale / c folded into the b_i.  Horner's scheme: four
// multiply-adds after the square; tile_row_exp_half_cap takes the same steps per score in
// paired instructions (each lane rounded as here), so this is the value it gives that score
// before subtracting the reference max.  b4 > 0, so s = -inf (a masked score) gives -inf.
__device__ __forceinline__ float cap_poly_at(float s, const FwdParams& p) {
  const float w = s * s;
  float t = fmaf(p.cap_poly[4], w, p.cap_poly[3]);
  t = fmaf(t, w, p.cap_poly[2]);
  t = fmaf(t, w, p.cap_poly[1]);
  t = fmaf(t, w, p.cap_poly[0]);
  return t * s;
}

// Soft-cap, in place, outside the polynomial's range: every raw score of the row becomes its
// base-2 capped score c log2(e) tanh(s scale / c) by the identity
// tanh(y) = 1 - 2 / (e^(2y) + 1) on ex2 and rcp (a masked NaN stays NaN).
__device__ __forceinline__ void cap_row_exact(uint32_t (&s)[128], const FwdParams& p) {
#pragma unroll
  for (int c = 0; c < 128; ++c)
    s[c] = __float_as_uint(p.cap_log2 * tanh_via_ex2(f32(s[c]) * p.cap_scale));
}

// Masked columns (outside [c_lo, c_hi]) of one tile row become `bits` (-inf by default).
__device__ __forceinline__ void mask_row(uint32_t (&s)[128], int c_lo, int c_hi,
                                         uint32_t bits = kNegInfBits) {
#pragma unroll
  for (int c = 0; c < 128; ++c)
    if ((unsigned)(c - c_lo) > (unsigned)(c_hi - c_lo)) s[c] = bits;
}

// ALiBi: the row's scores become base-2 biased scores in place,
// scale * s * log2(e) - slope2 * |drow - c| with drow the row's offset from the tile's first
// key and slope2 the head's slope times log2(e); -inf (masked) stays -inf.
__device__ __forceinline__ void alibi_row(uint32_t (&s)[128], const FwdParams& p, float slope2,
                                          float drow) {
#pragma unroll
  for (int c = 0; c < 128; c += 2) {
    const float d0 = fabsf(drow - (float)c), d1 = fabsf(drow - (float)(c + 1));
    float t0, t1;
    ffma2(t0, t1, f32(s[c]), f32(s[c + 1]), p.kscale, p.kscale, -slope2 * d0, -slope2 * d1);
    s[c] = __float_as_uint(t0);
    s[c + 1] = __float_as_uint(t1);
  }
}

// Soft-capped P = 2^(cap(s) - m_use) for one 64-column half of a tile row of raw scores
// (every |s| <= cap_fast_max, masked ones -inf): the polynomial of cap_poly_at with the
// subtraction of m_use folded into its last step, so the cap costs the FMA pipe five paired
// instructions per pair of scores on top of the plain exponential.  A masked score's -inf
// stays -inf through the polynomial (positive leading coefficient), so its exponential is 0.
// Returns the half's sum.
__device__ __forceinline__ float tile_row_exp_half_cap(const uint32_t (&s)[128], int base,
                                                       const FwdParams& p, float m_use,
                                                       uint32_t (&pk)[32]) {
  const float b0 = p.cap_poly[0], b1 = p.cap_poly[1], b2 = p.cap_poly[2], b3 = p.cap_poly[3],
              b4 = p.cap_poly[4];
  float a0 = 0.f, a1 = 0.f, c0 = 0.f, c1 = 0.f;
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    const float s0 = f32(s[base + c]), s1 = f32(s[base + c + 1]);
    float w0, w1, t0, t1;
    fmul2(w0, w1, s0, s1, s0, s1);
    ffma2(t0, t1, w0, w1, b4, b4, b3, b3);
    ffma2(t0, t1, t0, t1, w0, w1, b2, b2);
    ffma2(t0, t1, t0, t1, w0, w1, b1, b1);
    ffma2(t0, t1, t0, t1, w0, w1, b0, b0);
    ffma2(t0, t1, t0, t1, s0, s1, -m_use, -m_use);   // cap(s) - m_use
    const float e0 = ex2_approx(t0);
    const float e1 = ex2_approx(t1);
    if ((c >> 1) & 1)
      add2(c0, c1, e0, e1);
    else
      add2(a0, a1, e0, e1);
    pk[c >> 1] = pack_bf16x2(e0, e1);
  }
  return (a0 + a1) + (c0 + c1);
}

// FP8 path: 2^(x - m_use + 6) = 64 P for one 64-column half of a tile row, packed four
// per TMEM column as E4M3 (key 4c + i in byte i of column c); returns the half's fp32 sum
// of P (the sum of 64 P divided by 64, exact).
__device__ __forceinline__ float tile_row_exp_half_e4m3(const uint32_t (&s)[128], int base,
                                                        float ks, float m_use,
                                                        uint32_t (&pk)[16]) {
  const float mu = m_use - 6.0f;
  float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
  for (int c = 0; c < 64; c += 4) {
    float x0, x1, x2, x3;
    ffma2(x0, x1, f32(s[base + c]), f32(s[base + c + 1]), ks, ks, -mu, -mu);
    ffma2(x2, x3, f32(s[base + c + 2]), f32(s[base + c + 3]), ks, ks, -mu, -mu);
    const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
    const float e2 = ex2_approx(x2), e3 = ex2_approx(x3);
    if ((c >> 2) & 1) {
      add2(b0, b1, e0, e1);
      add2(b0, b1, e2, e3);
    } else {
      add2(a0, a1, e0, e1);
      add2(a0, a1, e2, e3);
    }
    pk[c >> 2] = pack_e4m3x4(e0, e1, e2, e3);
  }
  return (((a0 + a1) + (b0 + b1)) * (1.0f / 64.0f));
}

// P = 2^(x ks - m_use) for one 64-column half of a tile row (x the raw score, or the
// base-2 score itself with ks = 1), packed as bf16 pairs; returns the half's fp32 sum (four
// independent packed accumulators).
__device__ __forceinline__ float tile_row_exp_half(const uint32_t (&s)[128], int base, float ks,
                                                   float m_use, uint32_t (&pk)[32]) {
  float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f, c0 = 0.f, c1 = 0.f, d0 = 0.f, d1 = 0.f;
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    float x0, x1;
    ffma2(x0, x1, f32(s[base + c]), f32(s[base + c + 1]), ks, ks, -m_use, -m_use);
    const float e0 = ex2_approx(x0);
    const float e1 = ex2_approx(x1);
    switch ((c >> 1) & 3) {
      case 0: add2(a0, a1, e0, e1); break;
      case 1: add2(b0, b1, e0, e1); break;
      case 2: add2(c0, c1, e0, e1); break;
      default: add2(d0, d1, e0, e1); break;
    }
    pk[c >> 1] = pack_bf16x2(e0, e1);
  }
  return ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
}

// K/V tiles [a, b] (relative to the unit's first tile jt0) that query tile t must visit; n = 0
// when the tile has no valid row.  make_pair_work turns them into the unit's steps that
// visit them (the same numbers, or mirrored when the steps run last tile first).
struct TileRange {
  int a, b, n;
};

__device__ __forceinline__ TileRange tile_range(const FwdParams& p, int tq0, int jt0,
                                                int n_tiles) {
  TileRange r{0, -1, 0};
  if (tq0 >= p.Nq || n_tiles == 0) return r;
  int lo, hi, lo2, hi2;
  row_interval(p.mask, tq0, lo, hi);
  row_interval(p.mask, min(tq0 + kBM, p.Nq) - 1, lo2, hi2);
  if (hi2 < lo) return r;
  r.a = lo / kBN - jt0;
  r.b = hi2 / kBN - jt0;
  r.n = r.b - r.a + 1;
  return r;
}

// One unit of work for the CTA's two query tiles t = 0, 1: query head h[t], rows
// [q0[t], q0[t] + 128) of batch entry b, the K/V tiles the two visit, [jt0, jt0 + n_tiles),
// and each tile's own sub-range of them.  Two layouts:
//   * adjacent tiles (the default): one head, rows [256 pair, 256 pair + 256);
//   * a head pair (GQA with an even group size): query heads 2m and 2m + 1 of one KV group
//     at the same 128 rows, so both tiles see the same keys under the same mask and every
//     K/V tile the CTA loads feeds both.
struct PairWork {
  int b, hk, h[2], q0[2], jt0, n_tiles;
  TileRange rng[2];
};

__device__ __forceinline__ PairWork make_pair_work(const FwdParams& p, int bh, int pair) {
  PairWork w;
  int q_first, q_span;
  if (p.head_pairs) {
    const int hp = p.Hq >> 1;
    w.b = bh / hp;
    w.h[0] = 2 * (bh % hp);
    w.h[1] = w.h[0] + 1;
    q_first = pair * kBM;
    w.q0[0] = w.q0[1] = q_first;
    q_span = kBM;
  } else {
    w.b = bh / p.Hq;
    w.h[0] = w.h[1] = bh % p.Hq;
    q_first = pair * 2 * kBM;
    w.q0[0] = q_first;
    w.q0[1] = q_first + kBM;
    q_span = 2 * kBM;
  }
  w.hk = w.h[0] / p.G;
  const int q_last = min(q_first + q_span - 1, p.Nq - 1);
  int lo_a, hi_a, lo_b, hi_b;
  row_interval(p.mask, q_first, lo_a, hi_a);
  row_interval(p.mask, q_last, lo_b, hi_b);
  w.jt0 = 0;
  w.n_tiles = 0;
  if (hi_b >= lo_a && p.Nk > 0) {
    w.jt0 = lo_a / kBN;
    w.n_tiles = hi_b / kBN - w.jt0 + 1;
  }
  w.rng[0] = tile_range(p, w.q0[0], w.jt0, w.n_tiles);
  w.rng[1] = tile_range(p, w.q0[1], w.jt0, w.n_tiles);
  // p.kv_reverse: steps run from the last K/V tile to the first (step j takes tile
  // jt0 + n_tiles - 1 - j, kv_tile_of_step), and each range becomes the steps that visit it.
  // The tiles nearest the diagonal come first: under ALiBi they hold the row maxima, so the
  // running max is set at once and O is hardly ever rescaled.
  if (p.kv_reverse)
    for (int t = 0; t < 2; ++t)
      if (w.rng[t].n > 0) {
        const int a = w.rng[t].a, b = w.rng[t].b;
        w.rng[t].a = w.n_tiles - 1 - b;
        w.rng[t].b = w.n_tiles - 1 - a;
      }
  return w;
}

// Absolute index of the K/V tile that step j of unit w visits.
__device__ __forceinline__ int kv_tile_of_step(const FwdParams& p, const PairWork& w, int j) {
  return p.kv_reverse ? w.jt0 + w.n_tiles - 1 - j : w.jt0 + j;
}

// The CTA's sequence of query pairs (the grid is persistent: one CTA per SM).  Unit u of a
// head combines pair P-1-k with pair k (k = u mod ceil(P/2)): under a causal mask their
// costs add up to the same total for every k, so handing units to CTAs round-robin
// balances the work, and consecutive units share a head, so the K/V tiles of the heads in
// flight stay in L2.  f returns false to stop (abort).
template <typename F>
__device__ __forceinline__ void for_each_pair(const FwdParams& p, const int* sched, F&& f) {
  const int P = p.num_pairs;
  if (p.sched) {
    // the CTA's own list, built at kernel start (build_schedule): one query pair per entry
    const int n = sched[0];
    for (int i = 0; i < n; ++i) {
      const int u = sched[1 + i];
      if (!f(u / P, u % P)) return;
    }
    return;
  }
  const int upb = (P + 1) / 2;
  const long long total = (long long)p.B * (p.head_pairs ? p.Hq / 2 : p.Hq) * upb;
  for (long long u = blockIdx.x; u < total; u += gridDim.x) {
    const int bh = (int)(u / upb);
    const int k = (int)(u % upb);
    if (!f(bh, P - 1 - k)) return;
    if (k != P - 1 - k && !f(bh, k)) return;
  }
}

// Cost-ordered deal of the work units (one query pair or head pair each) for masks under
// which the units' costs follow the data (packed documents).  Every CTA computes the same
// thing: the cost of every unit (the K/V tiles it visits, plus one for its fill and
// epilogue), a sort by descending cost (ties by index, so the order is the same in every
// CTA), and a snake deal of the sorted units -- CTA c takes sorted positions c and
// 2 G - 1 - c of every 2 G, G the grid -- which gives each CTA one of the heaviest and one of
// the lightest of each round (within 2 % of the longest-first greedy deal on the packed-
// document workload, against 20 % above the mean for dealing in index order).  keys is
// scratch shared memory for the sort; the CTA's list goes to sched[0] (count), sched[1..],
// in index order.
__device__ __forceinline__ void build_schedule(const FwdParams& p, uint32_t* keys, int* sched) {
  const int P = p.num_pairs;
  const int U = p.B * (p.head_pairs ? p.Hq / 2 : p.Hq) * P;
  int Up = 1;
  while (Up < U) Up <<= 1;
  for (int u = threadIdx.x; u < Up; u += kThreads) {
    uint32_t key = 0xffffffffu;
    if (u < U) {
      const PairWork w = make_pair_work(p, u / P, u % P);
      key = ((uint32_t)(0xffff - min(w.n_tiles + 1, 0xffff)) << 16) | (uint32_t)u;
    }
    keys[u] = key;
  }
  __syncthreads();
  // bitonic sort, ascending keys = descending cost, then ascending unit index
  for (int k = 2; k <= Up; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < Up; i += kThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint32_t a = keys[i], b = keys[ixj];
          if ((a > b) == ((i & k) == 0)) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  const int G = (int)gridDim.x, c = (int)blockIdx.x, G2 = 2 * G;
  for (int r = threadIdx.x; r < U; r += kThreads) {
    const int m = r % G2;
    if (m == c || m == G2 - 1 - c) sched[1 + 2 * (r / G2) + (m >= G ? 1 : 0)] = (int)(keys[r] & 0xffffu);
  }
  __syncthreads();
  // The CTA runs its units in index order (head-major, query rows ascending), not in cost
  // order: every CTA then moves through the heads at about the same pace, and a document's
  // K/V tiles are read by its query tiles while they are still in L2 (in cost order the
  // query tiles of one document run at scattered times and their K/V comes from DRAM again).
  if (threadIdx.x == 0) {
    const int rem = U % G2;
    const int n = 2 * (U / G2) + (rem > c ? 1 : 0) + (rem > G2 - 1 - c ? 1 : 0);
    sched[0] = n;
    for (int i = 2; i <= n; ++i) {           // insertion sort of sched[1..n], n <= kSchedMax
      const int v = sched[i];
      int j = i - 1;
      while (j >= 1 && sched[j] > v) {
        sched[j + 1] = sched[j];
        --j;
      }
      sched[j + 1] = v;
    }
  }
  // the K/V ring's copies will overwrite the keys through the async proxy
  fence_proxy_async_smem();
  __syncthreads();
}

template <int D, bool kAlibi, bool kFp8, bool kCap>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = Cfg<D, kFp8>;
  constexpr int NS = C::kStages;
  static_assert(!(kFp8 && (kAlibi || D != 128)), "FP8 path: d = 128, no bias");
  static_assert(!(kCap && (kFp8 || kAlibi)), "soft-cap: bf16 path without bias");
  // FP8: the lazy-rescale bound is 2^2 and P is stored as E4M3 of 64 P (<= 256 < 448), so
  // probabilities down to 2^-12 of the reference stay in E4M3's normal range.
  constexpr float kThreshold = kFp8 ? 2.0f : kRescaleThreshold;
  constexpr float kPScale = 64.0f;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);
  const uint32_t sQ = base_u32 + C::kQOff;
  const uint32_t sRing = base_u32 + C::kRingOff;
  const uint32_t sBar = base_u32 + C::kBarOff;
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * (uint32_t)i; };
  // Q_t loaded, Q_t free (its last QK^T done), K/V ring full/empty, S_t ready, P_t ready,
  // O_t final, all MMAs done.
  const int BAR_Q = 0, BAR_QF = 2, BAR_FULL = 4, BAR_EMPTY = 4 + NS, BAR_S = 4 + 2 * NS,
            BAR_P = 6 + 2 * NS, BAR_O = 10 + 2 * NS, BAR_DONE = 12 + 2 * NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::kBarOff + C::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(BAR_Q + t), 1);
      mbar_init(bar(BAR_QF + t), 1);
      mbar_init(bar(BAR_S + t), 1);
      mbar_init(bar(BAR_P + 2 * t), 4);
      mbar_init(bar(BAR_P + 2 * t + 1), 4);
      mbar_init(bar(BAR_O + t), 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(BAR_FULL + s), 1);
      mbar_init(bar(BAR_EMPTY + s), 1);
    }
    mbar_init(bar(BAR_DONE), 1);
    *abort_flag = 0;
    init_wait_limit(abort_flag, p.err);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int* sched = reinterpret_cast<int*>(base + C::kSchedOff);
  if (p.sched) build_schedule(p, reinterpret_cast<uint32_t*>(base + C::kRingOff), sched);

  if (warp >= kMmaWarp) {
   regs_decrease<kCap ? kRegsOtherCap : kRegsOther>();
   if (warp == kTmaWarp) {
    // ------------------------------------------------------------ K/V TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0;          // ring loads issued so far, across all pairs
      for_each_pair(p, sched, [&](int bh, int pair) -> bool {
        const PairWork w = make_pair_work(p, bh, pair);
        const int zkv = w.b * p.Hkv + w.hk;
        for (int i = 0; i < 2 * w.n_tiles; ++i) {
          const int s = issued % NS;
          const int round = issued / NS;
          if (round > 0 &&
              !mbar_wait(bar(BAR_EMPTY + s), (round - 1) & 1, abort_flag, p.err, kSiteEmpty))
            return false;
          mbar_arrive_expect_tx(bar(BAR_FULL + s), C::kTileBytes);
          const int row = kv_tile_of_step(p, w, i >> 1) * kBN;
          const CUtensorMap* m = (i & 1) ? &tmV : &tmK;
          if (kFp8 && (i & 1)) {
            // FP8 V is stored transposed ([d][keys] per head): one box of d rows x 128 keys
            tma_load_3d(sRing + s * C::kTileBytes, m, bar(BAR_FULL + s), row, 0, zkv);
          } else {
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d(sRing + s * C::kTileBytes + c * C::kChunkBytes, m, bar(BAR_FULL + s),
                          c * (128 / C::kElem), row, zkv);
          }
          ++issued;
        }
        return true;
      });
      // Outstanding copies must land before the CTA may exit (matters only on abort).
      for (int s = 0; s < NS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / NS) * NS;
        mbar_wait(bar(BAR_FULL + s), (last / NS) & 1, nullptr, p.err, kSiteDrain);
      }
    }
    __syncwarp();
   } else if (warp == kQWarp) {
    // -------------------------------------------------------------- Q TMA producer
    // Each query tile's Q is reloaded as soon as the previous pair's last QK^T of that
    // tile has completed, independently of the K/V ring.
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      int pairs = 0;
      int loads[2] = {0, 0};   // Q loads issued per query tile (they differ after an abort)
      for_each_pair(p, sched, [&](int bh, int pair) -> bool {
        const PairWork w = make_pair_work(p, bh, pair);
        for (int t = 0; t < 2; ++t) {
          if (pairs > 0 &&
              !mbar_wait(bar(BAR_QF + t), (pairs - 1) & 1, abort_flag, p.err, kSiteQFree))
            return false;
          mbar_arrive_expect_tx(bar(BAR_Q + t), C::kTileBytes);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(sQ + t * C::kTileBytes + c * C::kChunkBytes, &tmQ, bar(BAR_Q + t),
                        c * (128 / C::kElem), w.q0[t], w.b * p.Hq + w.h[t]);
          ++loads[t];
        }
        ++pairs;
        return true;
      });
      // The last load of each tile must land before the CTA may exit.
      for (int t = 0; t < 2; ++t)
        if (loads[t] > 0)
          mbar_wait(bar(BAR_Q + t), (loads[t] - 1) & 1, nullptr, p.err, kSiteDrain);
    }
    __syncwarp();
   } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- tcgen05 issuer
    // The whole warp runs this role with warp-uniform values and one elected lane issues
    // each tensor-core operation, so descriptors stay in the uniform datapath.
    {
      constexpr uint32_t idesc_qk =
          kFp8 ? idesc_e4m3_f32(kBM, kBN) : idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = kFp8 ? idesc_e4m3_f32(kBM, D) : idesc_bf16_f32(kBM, D, true);
      // Descriptors differ only in their start-address field (address >> 4, 14 bits; the
      // CTA's shared memory stays below 2^18 bytes, so adding an offset never carries out
      // of it): keep three base descriptors and add offsets in 16-byte units.
      const uint64_t dQ = smem_desc(sQ, 16, 1024);
      const uint64_t dK = smem_desc(sRing, 16, 1024);
      // bf16 V is MN-major (d along the 128-byte rows); FP8 V^T is K-major like K
      const uint64_t dV = kFp8 ? smem_desc(sRing, 16, 1024) : smem_desc(sRing, C::kChunkBytes, 1024);
      auto issue_qk = [&](int t, int sk) {
        const uint32_t d_tmem = tmem + 128u * t;
        const uint32_t q_off = (uint32_t)(t * C::kTileBytes) >> 4;
        const uint32_t k_off = (uint32_t)(sk * C::kTileBytes) >> 4;
        // one k-step reads 32 bytes of every row: 16 bf16 or 32 E4M3 values
#pragma unroll
        for (int kk = 0; kk < D * C::kElem / 32; ++kk) {
          const uint32_t off = ((kk >> 2) * C::kChunkBytes + (kk & 3) * 32) >> 4;
          if constexpr (kFp8)
            umma_ss_f8_warp(d_tmem, dQ + q_off + off, dK + k_off + off, idesc_qk, kk > 0 ? 1u : 0u);
          else
            umma_ss_warp(d_tmem, dQ + q_off + off, dK + k_off + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t[:, 64h : 64h + 64] V_j[64h : 64h + 64]: key half h of the PV product.
      auto issue_pv_half = [&](int t, int sv, int h, bool first) {
        const uint32_t d_tmem = tmem + 256u + 128u * t;
        const uint32_t v_off = (uint32_t)(sv * C::kTileBytes) >> 4;
        if constexpr (kFp8) {
          // E4M3 P: four keys per TMEM column in S columns [96, 128); a k-step is 32 keys
          const uint32_t a_tmem = tmem + 128u * t + 96u;
#pragma unroll
          for (int k = 0; k < kBN / 64; ++k) {
            const int kk = h * (kBN / 64) + k;
            umma_ts_f8_warp(d_tmem, a_tmem + 8u * kk, dV + v_off + ((kk * 32) >> 4), idesc_pv,
                            (!first || kk > 0) ? 1u : 0u);
          }
        } else {
          const uint32_t a_tmem = tmem + 128u * t + 64u;
#pragma unroll
          for (int k = 0; k < kBN / 32; ++k) {
            const int kk = h * (kBN / 32) + k;
            umma_ts_warp(d_tmem, a_tmem + 8u * kk, dV + v_off + ((kk * 16 * 128) >> 4), idesc_pv,
                         (!first || kk > 0) ? 1u : 0u);
          }
        }
      };
      int pairs = 0;        // pairs started
      int kv = 0;           // ring index of the next K tile
      int pcount0 = 0, pcount1 = 0;
      bool ok = true;
      // PV of union step jv for query tile t (a compile-time constant at every call), if t
      // visits it: wait for P, issue, and signal the epilogue after the tile's last PV.
      auto pv_for = [&](const TileRange& rg, int t, int& pcount, int jv, int sv) -> bool {
        if (jv < rg.a || jv > rg.b) return true;
        // The softmax hands P over in two key halves; the first half's product runs while
        // the second half is being computed.
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait_warp(bar(BAR_P + 2 * t + h), pcount & 1, abort_flag, p.err, kSitePFull))
            return false;
          tc_fence_after();
          issue_pv_half(t, sv, h, jv == rg.a);
        }
        ++pcount;
        if (jv == rg.b) umma_commit_warp(bar(BAR_O + t));
        return true;
      };
      for_each_pair(p, sched, [&](int bh, int pair) -> bool {
        const PairWork w = make_pair_work(p, bh, pair);
        const TileRange r0 = w.rng[0], r1 = w.rng[1];
        if (!mbar_wait_warp(bar(BAR_Q + 0), pairs & 1, abort_flag, p.err, kSiteQ)) return ok = false;
        if (!mbar_wait_warp(bar(BAR_Q + 1), pairs & 1, abort_flag, p.err, kSiteQ)) return ok = false;
        ++pairs;
        tc_fence_after();
        if (r0.n == 0) umma_commit_warp(bar(BAR_QF + 0));
        if (r1.n == 0) umma_commit_warp(bar(BAR_QF + 1));
        const int n = w.n_tiles;
        for (int j = 0; j < n; ++j) {
          const int ik = kv + 2 * j;
          const int sk = (int)((unsigned)ik % (unsigned)NS);
          if (!mbar_wait_warp(bar(BAR_FULL + sk), ((unsigned)ik / NS) & 1, abort_flag, p.err, kSiteFullK))
            return ok = false;
          tc_fence_after();
          int sv = 0;
          if (j > 0) {
            const int iv = ik - 1;
            sv = (int)((unsigned)iv % (unsigned)NS);
            if (!mbar_wait_warp(bar(BAR_FULL + sv), ((unsigned)iv / NS) & 1, abort_flag, p.err, kSiteFullV))
              return ok = false;
            tc_fence_after();
          }
          // Per query tile: PV of the previous step, then QK^T of this one.  In-order
          // tensor pipe: the QK^T overwrites S_t (and P_t inside it) only after the PV MMA
          // just issued has read P_t.
          if (j > 0 && !pv_for(r0, 0, pcount0, j - 1, sv)) return ok = false;
          if (j >= r0.a && j <= r0.b) {
            issue_qk(0, sk);
            umma_commit_warp(bar(BAR_S + 0));
            if (j == r0.b) umma_commit_warp(bar(BAR_QF + 0));
          }
          if (j > 0 && !pv_for(r1, 1, pcount1, j - 1, sv)) return ok = false;
          if (j >= r1.a && j <= r1.b) {
            issue_qk(1, sk);
            umma_commit_warp(bar(BAR_S + 1));
            if (j == r1.b) umma_commit_warp(bar(BAR_QF + 1));
          }
          if (j > 0) umma_commit_warp(bar(BAR_EMPTY + sv));
          umma_commit_warp(bar(BAR_EMPTY + sk));
        }
        if (n > 0) {
          const int iv = kv + 2 * n - 1;
          const int sv = (int)((unsigned)iv % (unsigned)NS);
          if (!mbar_wait_warp(bar(BAR_FULL + sv), ((unsigned)iv / NS) & 1, abort_flag, p.err, kSiteFullV))
            return ok = false;
          tc_fence_after();
          if (!pv_for(r0, 0, pcount0, n - 1, sv)) return ok = false;
          if (!pv_for(r1, 1, pcount1, n - 1, sv)) return ok = false;
          umma_commit_warp(bar(BAR_EMPTY + sv));
        }
        kv += 2 * n;
        return true;
      });
      // Every MMA issued above must be complete before TMEM is released.
      umma_commit_warp(bar(BAR_DONE));
      mbar_wait_warp(bar(BAR_DONE), 0, nullptr, p.err, kSiteDrain);
    }
    __syncwarp();
   }
  } else {
    regs_increase<kCap ? kRegsSoftmaxCap : kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warpgroups
    const int t = warp >> 2;                 // query tile of this warpgroup
    const int wq = warp & 3;                 // TMEM lane quarter this warp may access
    const int r = wq * 32 + lane;            // row inside the tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128u * t;
    const uint32_t tP = tS + 64u;
    const uint32_t tO = tmem + lane_off + 256u + 128u * t;
    int scount = 0, ocount = 0;

    for_each_pair(p, sched, [&](int bh, int pair) -> bool {
      const PairWork w = make_pair_work(p, bh, pair);
      const TileRange rng = t ? w.rng[1] : w.rng[0];
      const int tq0 = w.q0[t];
      const int head = w.h[t];
      const int row = tq0 + r;
      int row_lo, row_hi;
      row_interval(p.mask, row, row_lo, row_hi);
      // ALiBi slope of this head in base-2 units (0: no bias).
      const float slope2 = kAlibi ? __ldg(p.alibi + head) * kLog2eF : 0.f;
      // FP8: the block scale of this query tile; a K tile's scale joins it per tile.
      const float qs = (kFp8 && tq0 < p.Nq)
                           ? __ldg(p.q_scales + (size_t)(w.b * p.Hq + head) * p.nqt + tq0 / kBM)
                           : 1.f;
      const float* ksc = kFp8 ? p.k_scales + (size_t)(w.b * p.Hkv + w.hk) * p.nkt : nullptr;
      // Tile-level bounds: a K/V tile needs no mask when every valid row of this query
      // tile sees every key of it and it lies inside Nk.
      int lo_last = 0, hi_first = 0;
      if (rng.n > 0) {
        int a0, a1;
        row_interval(p.mask, min(tq0 + kBM, p.Nq) - 1, lo_last, a0);
        row_interval(p.mask, tq0, a1, hi_first);
      }

      float m_ref = -INFINITY;   // reference max (log2 units) of the exponentials in O, l
      float l = 0.f;
      for (int i = 0; i < rng.n; ++i) {
        bool ok = mbar_wait(bar(BAR_S + t), scount & 1, abort_flag, p.err, kSiteSFull);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) return false;
        ++scount;
        tc_fence_after();
        uint32_t s[128];
        tmem_ld_x128(tS, s);
        const int k0 = kv_tile_of_step(p, w, rng.a + i) * kBN;
        const bool masked =
            !(lo_last <= k0 && k0 + kBN - 1 <= hi_first && k0 + kBN <= p.Nk);
        float mx;
        bool cap_fused = false;   // soft-cap folded into the exponentials (see below)
        const float ks_eff = kFp8 ? p.kscale * qs * __ldg(ksc + k0 / kBN) : p.kscale;
        if constexpr (kFp8) {
          const float mx_raw = masked ? tile_row_max<true>(s, row_lo - k0, row_hi - k0)
                                      : tile_row_max<false>(s, 0, 0);
          mx = mx_raw * ks_eff;
        } else if constexpr (kCap) {
          // When the row's raw scores (masked ones included) lie in the polynomial's range,
          // the cap (increasing) of the raw max over the visible columns is the row max of
          // the capped scores, and the cap itself is applied inside the exponential loop
          // (masked scores -inf).  Otherwise the scores become base-2 capped scores in place
          // by the ex2/rcp identity, then -inf where masked, then the row max.
          cap_fused = tile_row_absmax(s) <= p.cap_fast_max;
          if (cap_fused) {
            mx = masked ? tile_row_max<true>(s, row_lo - k0, row_hi - k0)
                        : tile_row_max<false>(s, 0, 0);
            if (mx != -INFINITY) mx = cap_poly_at(mx, p);
          } else {
            cap_row_exact(s, p);
            if (masked) mask_row(s, row_lo - k0, row_hi - k0);
            mx = tile_row_max<false>(s, 0, 0);
          }
        } else if constexpr (!kAlibi) {
          const float mx_raw = masked ? tile_row_max<true>(s, row_lo - k0, row_hi - k0)
                                      : tile_row_max<false>(s, 0, 0);
          mx = mx_raw * p.kscale;
        } else {
          // The bias changes the order of the scores, so the row max is taken over the
          // biased, base-2 scores themselves.
          if (masked) mask_row(s, row_lo - k0, row_hi - k0);
          alibi_row(s, p, slope2, (float)(row - k0));   // no soft-cap with ALiBi
          mx = tile_row_max<false>(s, 0, 0);
        }
        const float m_new = fmaxf(m_ref, mx);
        const bool need = m_new > m_ref + kThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_ref - m_new);
          m_ref = m_new;
        }
        if (i > 0 && __any_sync(0xffffffffu, need)) {
          // Rescale this row of O.  PV of the previous tile is complete: the commit that
          // signalled this S was issued after it.  The next PV is issued only after the
          // arrives below.
#pragma unroll 1
          for (int cc = 0; cc < D / 16; ++cc) {
            uint32_t o[16];
            tmem_ld_x16(tO + 16u * cc, o);
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(f32(o[k]) * alpha);
            tmem_st_x16(tO + 16u * cc, o);
          }
        }
        // P = 2^(x - m_ref) as bf16 pairs, written over the upper half of S in TMEM and
        // handed to the tensor core one 64-key half at a time.  Masked scores are -inf, so
        // their exponentials are exactly 0.
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        float sum = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if constexpr (kFp8) {
            uint32_t pk[16];
            sum += tile_row_exp_half_e4m3(s, 64 * half, ks_eff, m_use, pk);
            tmem_st_x16(tS + 96u + 16u * half, pk);
          } else {
            uint32_t pk[32];
            if constexpr (kAlibi) {
              sum += tile_row_exp_half(s, 64 * half, 1.f, m_use, pk);
            } else if constexpr (kCap) {
              if (cap_fused)
                sum += tile_row_exp_half_cap(s, 64 * half, p, m_use, pk);
              else
                sum += tile_row_exp_half(s, 64 * half, 1.f, m_use, pk);   // capped in place
            } else {
              sum += tile_row_exp_half(s, 64 * half, p.kscale, m_use, pk);
            }
            tmem_st_x32(tP + 32u * half, pk);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_P + 2 * t + half));
        }
        l = l * alpha + sum;
      }
      if (rng.n == 0) return true;   // no valid row in this query tile

      // Epilogue.  Reading O here, before this warpgroup's next arrive on P, orders it
      // before the next pair's first PV (which overwrites O).
      bool ok = mbar_wait(bar(BAR_O + t), ocount & 1, abort_flag, p.err, kSiteOFinal);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) return false;
      ++ocount;
      tc_fence_after();
      const bool valid = row < p.Nq;
      // FP8: O holds 64 P V_codes; the V scale of the head and the 64 come out here
      const float o_mul = kFp8 ? __ldg(p.v_scales + w.b * p.Hkv + w.hk) / kPScale : 1.f;
      const float inv_l = (l > 0.f) ? o_mul / l : 0.f;
      const float lse = (l > 0.f) ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
      const size_t row_index = (size_t)(w.b * p.Hq + head) * (size_t)p.Nq + (size_t)row;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + row_index * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld_x32(tO + 32u * cc, o);
        uint32_t wv[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          wv[k] = pack_bf16x2(f32(o[2 * k]) * inv_l, f32(o[2 * k + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * cc);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(wv[4 * k], wv[4 * k + 1], wv[4 * k + 2], wv[4 * k + 3]);
        }
      }
      if (valid) p.lse[row_index] = lse;
      tc_fence_before();
      return true;
    });
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Rows with no key at all (Nk == 0): O = 0 and LSE = -inf, the degenerate case of the
// definition (empty softmax).
__global__ void attn_fill_empty_kernel(__nv_bfloat16* o, float* lse, size_t rows, int D) {
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i < rows * (size_t)D) o[i] = __float2bfloat16(0.f);
  if (i < rows) lse[i] = -INFINITY;
}

template <int D, bool kAlibi, bool kFp8 = false, bool kCap = false>
int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const FwdParams& p, cudaStream_t stream) {
  using C = Cfg<D, kFp8>;
  static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_sm100_kernel<D, kAlibi, kFp8, kCap>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return -4;
  const long long per_head = p.sched ? p.num_pairs : (p.num_pairs + 1) / 2;
  const long long units = per_head * p.B * (p.head_pairs ? p.Hq / 2 : p.Hq);
  const long long grid = units < p.num_sms ? units : p.num_sms;
  attn_fwd_sm100_kernel<D, kAlibi, kFp8, kCap>
      <<<(unsigned)grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace

// One kernel per combination of hooks, so that each carries only its own softmax code (the
// unrolled per-row loops are long, and a kernel holding several variants ran slower).
int launch_attn_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const FwdParams& p, int d, cudaStream_t stream) {
  const bool alibi = p.alibi != nullptr;
  const bool cap = p.softcap > 0.f;
  if (p.q_scales != nullptr) return d == 128 ? launch_fwd<128, false, true>(tq, tk, tv, p, stream) : -2;
  if (alibi && cap) return -2;
  if (d == 128) return alibi ? launch_fwd<128, true>(tq, tk, tv, p, stream)
                       : cap ? launch_fwd<128, false, false, true>(tq, tk, tv, p, stream)
                             : launch_fwd<128, false>(tq, tk, tv, p, stream);
  if (d == 64) return alibi ? launch_fwd<64, true>(tq, tk, tv, p, stream)
                      : cap ? launch_fwd<64, false, false, true>(tq, tk, tv, p, stream)
                            : launch_fwd<64, false>(tq, tk, tv, p, stream);
  return -2;
}

int launch_fill_empty(void* o, float* lse, size_t rows, int d, cudaStream_t stream) {
  const size_t n = rows * (size_t)d;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (blocks == 0) return 0;
  attn_fill_empty_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<__nv_bfloat16*>(o), lse,
                                                     rows, d);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace attn
