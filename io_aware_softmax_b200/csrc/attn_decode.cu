// Split-KV decode attention for sm_100a (FlashDecoding, "3.7 어텐션 II", section 3.7.4):
// one query token per sequence against a long KV cache, either contiguous or paged with a
// page table and per-sequence lengths (PagedAttention-style in-flight batching, sections
// 3.7.4 and 3.7.8).  The cache axis T is cut
// into S splits; every split runs the online softmax over its slice and emits a partial
// (O normalised by its own sum, natural-log LSE); a second kernel merges the splits with the
// rescaling rule  L = max_s LSE_s, w_s = exp(LSE_s - L), O = sum w_s O_s / sum w_s,
// LSE = L + ln(sum w_s).
//
// The work is HBM-bound (each cache byte is used by only G = Hq/Hkv query rows), so the
// kernel is built around moving bytes: one CTA handles all G query heads of a KV head (GQA:
// the cache is read once per group, never replicated -- "3.7 어텐션 II", section 3.7.5),
// a persistent grid of (SM count x resident CTAs) walks the (batch, kv-head, split) items,
// and a producer warp keeps a 3-stage ring of 64-token K/V tiles in flight with TMA loads
// (128B-swizzled, each CTA loading only into its own shared memory).  The four consumer
// warps each take 16 tokens of a stage.
// The two small products per 16 tokens (scores = q K^T with the G rows padded to 16, and
// O += P V) use warp-level mma.sync so that the SM's issue slots stay free for the memory
// pipeline; the tensor work is a few percent of what the tensor cores could do in the time
// the bytes take to arrive.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace {

constexpr int kTok = 64;          // tokens per stage
constexpr int kStagesDec = 3;
constexpr int kConsumerWarps = 4;
constexpr int kDecThreads = (kConsumerWarps + 1) * 32;
constexpr float kRescaleThresholdDec = 8.0f;
constexpr float kLn2 = 0.69314718055994531f;

enum : uint32_t { kSiteDecFull = 101, kSiteDecEmpty, kSiteDecDrain };

template <int D>
struct DecCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kChunkBytes = kTok * 128;            // 64 rows x 128 bytes
  static constexpr int kHalfBytes = kChunks * kChunkBytes;  // the K (or V) part of a stage
  static constexpr int kStageBytes = 2 * kHalfBytes;
  static constexpr int kRingBytes = kStagesDec * kStageBytes;
};

__host__ __device__ constexpr int dec_smem_bytes(int D, int G) {
  // ring + per-warp (m, l, O rows) scratch for the in-CTA merge + barriers, the abort flag
  // and the wait limit (with their 8-byte alignment) + alignment of the base
  return kStagesDec * 2 * (D / 64) * kTok * 128 + kConsumerWarps * G * (D + 2) * 4 + 96 + 1024;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of element (token, d) in a 128B-swizzled [64 tokens x D] stage half: d is cut
// into 64-wide chunks of 64 rows x 128 bytes; within a row the 16-byte unit index is XORed
// with (row mod 8) by the TMA swizzle.
__device__ __forceinline__ uint32_t swz_off(int tok, int d) {
  return (uint32_t)((d >> 6) * (kTok * 128) + tok * 128 + ((((d & 63) >> 3) ^ (tok & 7)) << 4));
}

// Item = (batch b, KV head hk, split s) and its rows [t0, t1).  The splits cut the rows at
// 64-row tile boundaries, as evenly as whole tiles allow: every tile is loaded by exactly
// one split (an uneven cut would load the tile across a boundary twice), and in a paged
// cache no tile straddles two pages (page_size is a multiple of the tile).  A paged
// sequence is cut at its own length.
template <bool kPaged>
__device__ __forceinline__ void item_coords(const DecParams& p, int item, int& b, int& hk, int& s,
                                            int& t0, int& t1) {
  const int bk = item / p.S;
  s = item % p.S;
  b = bk / p.Hkv;
  hk = bk % p.Hkv;
  int T = p.T;
  if (kPaged) {
    const long long cap = (long long)p.max_pages * p.page_size;
    T = (int)min(max((long long)__ldg(p.seq_lens + b), 0LL), cap);
  }
  const long long tiles = (T + kTok - 1) / kTok;
  t0 = (int)((s * tiles) / p.S) * kTok;
  t1 = (int)min((long long)T, (((s + 1) * tiles) / p.S) * kTok);
  if (t1 < t0) t1 = t0;
}

template <int D, bool kUpper, bool kPaged>
__global__ void __launch_bounds__(kDecThreads)
attn_decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const DecParams p, int G) {
  using C = DecCfg<D>;
  constexpr int NS = kStagesDec;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);
  const uint32_t sRing = base_u32;
  float* scr_o = reinterpret_cast<float*>(base + C::kRingBytes);      // [warp][G][D]
  float* scr_m = scr_o + kConsumerWarps * G * D;                       // [warp][G]
  float* scr_l = scr_m + kConsumerWarps * G;                           // [warp][G]
  const uint32_t sBar = (smem_u32(scr_l + kConsumerWarps * G) + 7u) & ~7u;
  auto full_bar = [&](int s) -> uint32_t { return sBar + 8u * s; };
  auto empty_bar = [&](int s) -> uint32_t { return sBar + 8u * (NS + s); };
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(base + (sBar - base_u32) + 8 * 2 * NS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kConsumerWarps);
    }
    *abort_flag = 0;
    init_wait_limit(abort_flag, p.err);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      uint32_t gi = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.num_items; item += gridDim.x) {
        int b, hk, s, t0, t1;
        item_coords<kPaged>(p, item, b, hk, s, t0, t1);
        const int n_st = (t1 - t0 + kTok - 1) / kTok;
        const int zc = b * p.Hkv + hk;
        for (int st = 0; st < n_st; ++st, ++gi) {
          const int sidx = gi % NS;
          const int round = gi / NS;
          if (round > 0 &&
              !mbar_wait(empty_bar(sidx), (round - 1) & 1, abort_flag, p.err, kSiteDecEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(sidx), C::kStageBytes);
          const uint32_t dst = sRing + sidx * C::kStageBytes;
          int row = t0 + st * kTok;
          int z = zc;
          if (kPaged) {
            // logical row -> (physical page, row in page); the cache map is
            // (d, page_size, num_pages * Hkv), so a page index outside the table's range
            // lands outside the map and reads zeros instead of faulting.
            const int page = __ldg(p.block_table + (size_t)b * p.max_pages + row / p.page_size);
            z = page * p.Hkv + hk;
            row = row % p.page_size;
          }
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
            tma_load_3d(dst + c * C::kChunkBytes, &tmK, full_bar(sidx), c * 64, row, z);
            tma_load_3d(dst + C::kHalfBytes + c * C::kChunkBytes, &tmV, full_bar(sidx), c * 64,
                        row, z);
          }
        }
      }
      // Outstanding copies must land before the CTA may exit.
      for (int s = 0; s < NS && (uint32_t)s < gi; ++s) {
        const uint32_t last = s + ((gi - 1 - s) / NS) * NS;
        mbar_wait(full_bar(s), (last / NS) & 1, nullptr, p.err, kSiteDecDrain);
      }
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------------- consumer warps
    const int w = warp;
    const int g = lane >> 2;       // accumulator row (and row + 8)
    const int tig = lane & 3;
    const int mi = lane >> 3;      // ldmatrix: which 8x8 matrix this lane addresses
    const int rr = lane & 7;       // ... and which row of it
    const __nv_bfloat16* qall = reinterpret_cast<const __nv_bfloat16*>(p.q);
    uint32_t gi = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.num_items; item += gridDim.x) {
      int b, hk, s, t0, t1;
      item_coords<kPaged>(p, item, b, hk, s, t0, t1);
      const int n_st = (t1 - t0 + kTok - 1) / kTok;
      const int qrow0 = b * p.Hq + hk * G;

      // q as the A operand (rows g and g + 8 of the 16-row padded group)
      uint32_t qa[D / 16][4];
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int col = 16 * kk + 2 * tig;
        const uint32_t* r0 = reinterpret_cast<const uint32_t*>(qall + (size_t)(qrow0 + g) * D);
        const uint32_t* r1 =
            reinterpret_cast<const uint32_t*>(qall + (size_t)(qrow0 + g + 8) * D);
        const bool v0 = g < G;
        const bool v1 = kUpper && (g + 8 < G);
        qa[kk][0] = v0 ? __ldg(r0 + col / 2) : 0u;
        qa[kk][1] = v1 ? __ldg(r1 + col / 2) : 0u;
        qa[kk][2] = v0 ? __ldg(r0 + col / 2 + 4) : 0u;
        qa[kk][3] = v1 ? __ldg(r1 + col / 2 + 4) : 0u;
      }
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      float o[D / 8][4];
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

      for (int st = 0; st < n_st; ++st, ++gi) {
        const int sidx = gi % NS;
        if (ok) {
          ok = mbar_wait(full_bar(sidx), (gi / NS) & 1, abort_flag, p.err, kSiteDecFull);
          ok = __all_sync(0xffffffffu, ok);
        }
        if (!ok) continue;
        const int tok0 = t0 + st * kTok + 16 * w;
        if (tok0 < t1) {
          const uint32_t kbase = sRing + sidx * C::kStageBytes;
          const uint32_t vbase = kbase + C::kHalfBytes;
          // scores for 16 tokens: two 8-token column tiles
          float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int tl = 16 * w + 8 * (mi >> 1) + rr;
            const int dd = 16 * kk + 8 * (mi & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kbase + swz_off(tl, dd), b0, b1, b2, b3);
            mma_bf16(sc[0], qa[kk], b0, b1);
            mma_bf16(sc[1], qa[kk], b2, b3);
          }
          float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int tok = tok0 + 8 * nt + 2 * tig + (e & 1);
              const int row = g + 8 * (e >> 1);
              float x = sc[nt][e] * p.kscale;
              if (tok >= t1 || row >= G) x = -INFINITY;
              sc[nt][e] = x;
              if (e < 2) mx0 = fmaxf(mx0, x); else mx1 = fmaxf(mx1, x);
            }
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
          const float mn0 = fmaxf(m0, mx0);
          if (mn0 > m0 + kRescaleThresholdDec) {
            const float a = ex2_approx(m0 - mn0);
            m0 = mn0;
            l0 *= a;
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) { o[nt][0] *= a; o[nt][1] *= a; }
          }
          if (kUpper) {
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn1 = fmaxf(m1, mx1);
            if (mn1 > m1 + kRescaleThresholdDec) {
              const float a = ex2_approx(m1 - mn1);
              m1 = mn1;
              l1 *= a;
#pragma unroll
              for (int nt = 0; nt < D / 8; ++nt) { o[nt][2] *= a; o[nt][3] *= a; }
            }
          }
          const float mu0 = (m0 == -INFINITY) ? 0.f : m0;
          const float mu1 = (m1 == -INFINITY) ? 0.f : m1;
          float pr[2][4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            pr[nt][0] = ex2_approx(sc[nt][0] - mu0);
            pr[nt][1] = ex2_approx(sc[nt][1] - mu0);
            l0 += pr[nt][0] + pr[nt][1];
            if (kUpper) {
              pr[nt][2] = ex2_approx(sc[nt][2] - mu1);
              pr[nt][3] = ex2_approx(sc[nt][3] - mu1);
              l1 += pr[nt][2] + pr[nt][3];
            } else {
              pr[nt][2] = 0.f;
              pr[nt][3] = 0.f;
            }
          }
          const uint32_t pa[4] = {pack_bf16x2(pr[0][0], pr[0][1]), pack_bf16x2(pr[0][2], pr[0][3]),
                                  pack_bf16x2(pr[1][0], pr[1][1]), pack_bf16x2(pr[1][2], pr[1][3])};
#pragma unroll
          for (int np = 0; np < D / 16; ++np) {
            const int tl = 16 * w + 8 * (mi & 1) + rr;
            const int dd = 16 * np + 8 * (mi >> 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_trans(vbase + swz_off(tl, dd), b0, b1, b2, b3);
            mma_bf16(o[2 * np], pa, b0, b1);
            mma_bf16(o[2 * np + 1], pa, b2, b3);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(sidx));
      }

      // ---- merge the four warps' partial states of this item
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      if (g < G) {
        if (tig == 0) {
          scr_m[w * G + g] = m0;
          scr_l[w * G + g] = l0;
        }
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
          float* dst = scr_o + ((size_t)w * G + g) * D + 8 * nt + 2 * tig;
          dst[0] = o[nt][0];
          dst[1] = o[nt][1];
        }
      }
      if (kUpper && g + 8 < G) {
        if (tig == 0) {
          scr_m[w * G + g + 8] = m1;
          scr_l[w * G + g + 8] = l1;
        }
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
          float* dst = scr_o + ((size_t)w * G + g + 8) * D + 8 * nt + 2 * tig;
          dst[0] = o[nt][2];
          dst[1] = o[nt][3];
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
      for (int idx = threadIdx.x; idx < G * D; idx += kConsumerWarps * 32) {
        const int r = idx / D;
        const int c = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kConsumerWarps; ++ww) M = fmaxf(M, scr_m[ww * G + r]);
        float out = 0.f, lse = -INFINITY;
        if (M != -INFINITY) {
          float wsum = 0.f, acc = 0.f;
#pragma unroll
          for (int ww = 0; ww < kConsumerWarps; ++ww) {
            const float wt = ex2_approx(scr_m[ww * G + r] - M);
            wsum += wt * scr_l[ww * G + r];
            acc += wt * scr_o[((size_t)ww * G + r) * D + c];
          }
          out = acc / wsum;
          lse = (M + log2f(wsum)) * kLn2;
        }
        const size_t prow = (size_t)(qrow0 + r) * p.S + s;
        p.o_part[prow * D + c] = out;
        if (c == 0) p.lse_part[prow] = lse;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    }
  }
  __syncthreads();
}

// One warp per (b, h) row: merge the S partial results of the split-KV kernel.
__global__ void attn_merge_kernel(const float* __restrict__ o_part,
                                  const float* __restrict__ lse_part, __nv_bfloat16* o,
                                  float* lse, long long rows, int S, int D) {
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* lp = lse_part + row * S;
  float M = -INFINITY;
  for (int s = lane; s < S; s += 32) M = fmaxf(M, lp[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  __nv_bfloat16* orow = o + row * D;
  if (M == -INFINITY) {
    for (int c = lane; c < D; c += 32) orow[c] = __float2bfloat16(0.f);
    if (lane == 0) lse[row] = -INFINITY;
    return;
  }
  float wsum = 0.f;
  for (int s = lane; s < S; s += 32) wsum += expf(lp[s] - M);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
  const float inv = 1.0f / wsum;
  for (int c = 4 * lane; c < D; c += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < S; ++s) {
      const float wt = expf(lp[s] - M);
      const float4 v = *reinterpret_cast<const float4*>(o_part + (row * S + s) * D + c);
      acc.x += wt * v.x;
      acc.y += wt * v.y;
      acc.z += wt * v.z;
      acc.w += wt * v.w;
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    *reinterpret_cast<__nv_bfloat162*>(orow + c) = lo;
    *reinterpret_cast<__nv_bfloat162*>(orow + c + 2) = hi;
  }
  if (lane == 0) lse[row] = M + logf(wsum);
}

template <int D, bool kUpper, bool kPaged>
int launch_split_t(const CUtensorMap& tk, const CUtensorMap& tv, const DecParams& p, int G,
                   int grid, cudaStream_t stream) {
  const int smem = dec_smem_bytes(D, G);
  if (cudaFuncSetAttribute(attn_decode_split_kernel<D, kUpper, kPaged>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return -4;
  attn_decode_split_kernel<D, kUpper, kPaged><<<grid, kDecThreads, smem, stream>>>(tk, tv, p, G);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

template <int D, bool kUpper>
int occupancy_t(int G) {
  const int smem = dec_smem_bytes(D, G);
  if (cudaFuncSetAttribute(attn_decode_split_kernel<D, kUpper, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, attn_decode_split_kernel<D, kUpper, false>,
                                                    kDecThreads, smem) != cudaSuccess || n < 1)
    return 1;
  return n;
}

}  // namespace

int decode_ctas_per_sm(int d, int G) {
  // Resident CTAs per SM for (d, G); the answer depends only on the kernel and its shared
  // memory, so it is computed once per (d, G) and device.
  static int cache[2][17][64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const int di = (d == 128) ? 1 : 0;
  if (G < 1 || G > 16 || dev < 0 || dev >= 64) return 1;
  int& slot = cache[di][G][dev];
  if (slot == 0) {
    if (d == 128) slot = G > 8 ? occupancy_t<128, true>(G) : occupancy_t<128, false>(G);
    else slot = G > 8 ? occupancy_t<64, true>(G) : occupancy_t<64, false>(G);
  }
  return slot;
}

int launch_decode_split(const CUtensorMap& tk, const CUtensorMap& tv, const DecParams& p, int d,
                        int G, int grid, cudaStream_t stream) {
  const bool paged = p.block_table != nullptr;
  if (d == 128) {
    if (paged)
      return G > 8 ? launch_split_t<128, true, true>(tk, tv, p, G, grid, stream)
                   : launch_split_t<128, false, true>(tk, tv, p, G, grid, stream);
    return G > 8 ? launch_split_t<128, true, false>(tk, tv, p, G, grid, stream)
                 : launch_split_t<128, false, false>(tk, tv, p, G, grid, stream);
  }
  if (d == 64) {
    if (paged)
      return G > 8 ? launch_split_t<64, true, true>(tk, tv, p, G, grid, stream)
                   : launch_split_t<64, false, true>(tk, tv, p, G, grid, stream);
    return G > 8 ? launch_split_t<64, true, false>(tk, tv, p, G, grid, stream)
                 : launch_split_t<64, false, false>(tk, tv, p, G, grid, stream);
  }
  return -2;
}

int launch_merge(const float* o_part, const float* lse_part, void* o, float* lse, long long rows,
                 int S, int d, cudaStream_t stream) {
  if (rows <= 0) return 0;
  const int warps = 4;
  const long long blocks = (rows + warps - 1) / warps;
  attn_merge_kernel<<<(unsigned)blocks, warps * 32, 0, stream>>>(
      o_part, lse_part, reinterpret_cast<__nv_bfloat16*>(o), lse, rows, S, d);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace attn
