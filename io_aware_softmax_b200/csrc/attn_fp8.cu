// FP8 (E4M3) inputs for the fused attention: block quantization with optional incoherent
// processing ("FlashAttention 논문 분석: IO-Aware Exact Attention", section "FP8 지원과 정확도
// 유지"): every block of `block_rows` rows of one (batch, head) gets its own scale
// (amax / 448, 448 being the largest finite E4M3 value), and Q and K may first be multiplied
// by the orthogonal matrix diag(signs) H / sqrt(d) (H the Sylvester Hadamard matrix), which
// leaves Q K^T unchanged and spreads outlier columns over all of d.
//
// Three kernels, each reading its input from HBM once where it can:
//  * rows (Q, K: row-major codes, blocks of at most 128 rows): a persistent grid; each block
//    arrives by tiled bulk tensor copies with the 128-byte swizzle, thread t holds row t in
//    registers (rotated there: the Hadamard butterflies need no other thread), the block's
//    amax is reduced, and the codes go back through shared memory to coalesced stores;
//  * vt (V: transposed codes [d][n_pad], one scale per head): a cluster of eight CTAs per
//    head; each CTA reduces the amax of its share of the head, the eight exchange it through
//    distributed shared memory, and each CTA then reads its share again (from L2) and writes
//    the transposed codes, staged in shared memory, with coalesced 16-byte stores;
//  * chunked (everything else: larger blocks, a rotated transposed output, unaligned outputs):
//    three launches over chunks of 64 rows of one (batch, head), 256 threads each, a warp per
//    8 consecutive rows, lane l holding columns [l d/32, (l + 1) d/32) and the butterflies
//    crossing lanes by shuffles:
//      1. amax: each chunk reduces the |values| of every block it touches in shared memory
//         and folds them into `scales` (zeroed first) with one atomic max per block;
//      2. quantize: x * (448 / amax) rounded to E4M3 (nearest even, saturating), written
//         row-major or transposed ([d][n_pad] per head, the K-major layout of V for the P V
//         product; columns [N, n_pad) zero);
//      3. finalize: scales = amax / 448 (1 for an all-zero block).
// All paths round every operation the same way (the butterflies in the same order, products
// by +-1 exact), so a row quantizes to the same bits whichever kernel takes it.
#include <algorithm>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace {

constexpr int kQuantThreads = 256;
constexpr int kChunkRows = 64;
constexpr int kRowsPerWarp = kChunkRows / (kQuantThreads / 32);   // 8
constexpr float kE4m3Max = 448.0f;

// 1 / sqrt(d) rounded to float (0.125 exactly for d = 64).
template <int D>
__device__ __forceinline__ constexpr float inv_sqrt_d() {
  return D == 128 ? 0.08838834764831845f : 0.125f;
}

// Multiplies this lane's d/32 values of a row by diag(signs) H / sqrt(d) (lane l holds
// columns [l d/32, (l + 1) d/32)).  Every operation is explicitly rounded, so each kernel that
// rotates a row produces the same bits (no FMA contraction that could differ between them).
template <int D>
__device__ __forceinline__ void rotate_row(const float* __restrict__ signs, float (&v)[D / 32]) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = __fmul_rn(v[e], __ldg(signs + lane * E + e));
  // Walsh-Hadamard butterflies: pairs (i, i ^ s) for s = 1, 2, ..., D / 2; the low index
  // gets a + b, the high one a - b.  Strides below E stay in the lane.
#pragma unroll
  for (int s = 1; s < E; s <<= 1)
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (!(e & s)) {
        const float a = v[e], b = v[e + s];
        v[e] = __fadd_rn(a, b);
        v[e + s] = __fsub_rn(a, b);
      }
  // Across lanes: the high lane of a pair gets o - v, the low one v + o, each as one fused
  // multiply-add by +-1 (exact product, one rounding: the same bits as the add or subtract).
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    const float sgn = (lane & s) ? -1.f : 1.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, v[e], s);
      v[e] = __fmaf_rn(sgn, v[e], o);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = __fmul_rn(v[e], inv_sqrt_d<D>());
}

// This lane's d/32 bf16 values at src as floats.
template <int D>
__device__ __forceinline__ void bf16_lane_values(const __nv_bfloat16* src, float (&v)[D / 32]) {
  if constexpr (D / 32 == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  } else {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src));
    v[0] = a.x; v[1] = a.y;
  }
}

// This lane's d/32 values of row `row` (zeros past the last row), rotated when signs != 0.
template <int D>
__device__ __forceinline__ void load_row(const __nv_bfloat16* __restrict__ x, long long row,
                                         bool valid, const float* __restrict__ signs,
                                         float (&v)[D / 32]) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  if (valid) {
    bf16_lane_values<D>(x + row * D + lane * E, v);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = 0.f;
  }
  if (signs != nullptr) rotate_row<D>(signs, v);
}

// Pass 1: per block, the largest |value| (after rotation) as float bits in amax_bits.
template <int D>
__global__ void __launch_bounds__(kQuantThreads)
quant_amax_kernel(const __nv_bfloat16* __restrict__ x, unsigned int* __restrict__ amax_bits,
                  int N, int block_rows, int nblk, int nchunk, const float* __restrict__ signs) {
  constexpr int E = D / 32;
  __shared__ unsigned int s_amax[kChunkRows + 2];   // blocks touched by this chunk
  const int bh = blockIdx.x / nchunk, chunk = blockIdx.x % nchunk;
  const int r0 = chunk * kChunkRows;
  const int b0 = r0 / block_rows;
  const int b1 = (min(r0 + kChunkRows, N) - 1) / block_rows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i <= b1 - b0; i += kQuantThreads) s_amax[i] = 0u;
  __syncthreads();
  const int w0 = r0 + warp * kRowsPerWarp;
  float v[kRowsPerWarp][E];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i)
    load_row<D>(x, (long long)bh * N + w0 + i, w0 + i < N, signs, v[i]);
  // one reduction per run of rows of the same block (a warp's 8 rows span at most two
  // blocks unless blocks are shorter than 8 rows)
  float run = 0.f;
  int run_blk = w0 / block_rows;
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int r = w0 + i;
    if (r >= N) break;
    const int blk = r / block_rows;
    if (blk != run_blk) {
      float m = run;
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
      if (lane == 0) atomicMax(&s_amax[run_blk - b0], __float_as_uint(m));
      run = 0.f;
      run_blk = blk;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) run = fmaxf(run, fabsf(v[i][e]));
  }
  if (w0 < N) {
    float m = run;
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
    if (lane == 0) atomicMax(&s_amax[run_blk - b0], __float_as_uint(m));   // non-negative
  }
  __syncthreads();
  for (int i = threadIdx.x; i <= b1 - b0; i += kQuantThreads)
    if (s_amax[i] != 0u) atomicMax(&amax_bits[(long long)bh * nblk + b0 + i], s_amax[i]);
}

// Pass 2: E4M3 codes.  Chunks cover max(N, n_pad) rows, so that a transposed output gets its
// zero columns [N, n_pad) from the same stores.
template <int D>
__global__ void __launch_bounds__(kQuantThreads)
quant_codes_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ out,
                   const unsigned int* __restrict__ amax_bits, int N, int block_rows, int nblk,
                   int nchunk, int transpose, int n_pad, int wide,
                   const float* __restrict__ signs) {
  constexpr int E = D / 32;
  const int bh = blockIdx.x / nchunk, chunk = blockIdx.x % nchunk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w0 = chunk * kChunkRows + warp * kRowsPerWarp;
  const int rows = transpose ? n_pad : N;
  // wide == 2 (transposed, n_pad % 16 == 0, output 16-byte aligned): the whole CTA stages
  // the chunk's codes in shared memory, so no warp may leave before the barrier
  if (w0 >= rows && wide != 2) return;
  // codes of column lane * E + e for the 8 rows, four rows per word (row 4k + j in byte j)
  uint32_t cw[E][2];
#pragma unroll
  for (int e = 0; e < E; ++e) cw[e][0] = cw[e][1] = 0u;
  float vv[kRowsPerWarp][E];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i)
    load_row<D>(x, (long long)bh * N + w0 + i, w0 + i < N, signs, vv[i]);
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int r = w0 + i;
    const float (&v)[E] = vv[i];
    float inv = 1.f;
    if (r < N) {
      const float amax =
          __uint_as_float(__ldg(amax_bits + (long long)bh * nblk + r / block_rows));
      inv = amax > 0.f ? kE4m3Max / amax : 1.f;
    }
#pragma unroll
    for (int e = 0; e < E; ++e)
      cw[e][i >> 2] |= (uint32_t)__nv_cvt_float_to_fp8(v[e] * inv, __NV_SATFINITE, __NV_E4M3)
                       << (8 * (i & 3));
  }
  auto code = [&](int i, int e) -> uint32_t {
    return (cw[e][i >> 2] >> (8 * (i & 3))) & 0xffu;
  };
  if (!transpose) {
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const int r = w0 + i;
      if (r >= N) break;
      uint8_t* dst = out + ((long long)bh * N + r) * D + lane * E;
      if constexpr (E == 4) {
        *reinterpret_cast<uint32_t*>(dst) =
            code(i, 0) | (code(i, 1) << 8) | (code(i, 2) << 16) | (code(i, 3) << 24);
      } else {
        *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(code(i, 0) | (code(i, 1) << 8));
      }
    }
    return;
  }
  if (wide == 2) {
    // Transposed through shared memory: column c of the chunk (64 rows = 64 bytes) sits at
    // words [17 c, 17 c + 16) (the odd stride spreads the columns over the banks); then each
    // thread writes whole 16-byte runs of a column, so a warp's stores cover whole columns.
    __shared__ uint32_t stage[D * 17];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int col = lane * E + e;
      stage[col * 17 + warp * 2] = cw[e][0];
      stage[col * 17 + warp * 2 + 1] = cw[e][1];
    }
    __syncthreads();
    for (int k = threadIdx.x; k < D * 4; k += kQuantThreads) {
      const int col = k >> 2, seg = k & 3;
      const int row0 = chunk * kChunkRows + 16 * seg;
      if (row0 >= n_pad) continue;
      const uint32_t* src = stage + col * 17 + seg * 4;
      *reinterpret_cast<uint4*>(out + ((long long)bh * D + col) * n_pad + row0) =
          make_uint4(src[0], src[1], src[2], src[3]);
    }
    return;
  }
  // transposed: column lane * E + e of the head holds rows [w0, w0 + 8) in 8 bytes
  uint8_t* base = out + (long long)bh * D * n_pad + w0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    uint8_t* dst = base + (long long)(lane * E + e) * n_pad;
    if (wide) {   // n_pad is a multiple of 8 and the output 8-byte aligned
      *reinterpret_cast<uint2*>(dst) = make_uint2(cw[e][0], cw[e][1]);
    } else {
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i)
        if (w0 + i < n_pad) dst[i] = (uint8_t)code(i, e);
    }
  }
}

constexpr uint32_t kSiteQuantLoad = 0x51u;
constexpr uint32_t kSiteQuantVt = 0x52u;

// ----------------------------------------------------------------------------- rows kernel
constexpr int kRowThreads = 128;                      // thread t <-> row t of a block
constexpr int kRowCtasPerSm = 2;
constexpr int kRowBufs = 3;                           // blocks in flight per CTA
constexpr uint32_t kRowBoxBytes = 128 * 128;          // one box: 128 rows x 64 bf16 columns

// Multiplies a whole row (held by one thread) by H / sqrt(d): the Walsh-Hadamard butterflies
// over pairs (i, i ^ s), s = 1, 2, ..., d / 2 in that order, the low index getting a + b and
// the high one a - b (pairs of pairs at once from s = 2 on).
template <int D>
__device__ __forceinline__ void hadamard_row(float (&v)[D]) {
#pragma unroll
  for (int e = 0; e < D; e += 2) {
    const float a = v[e], b = v[e + 1];
    v[e] = __fadd_rn(a, b);
    v[e + 1] = __fsub_rn(a, b);
  }
#pragma unroll
  for (int s = 2; s < D; s <<= 1)
#pragma unroll
    for (int e = 0; e < D; e += 2)
      if (!(e & s)) butterfly2(v[e], v[e + 1], v[e + s], v[e + s + 1]);
#pragma unroll
  for (int e = 0; e < D; e += 2) fmul2(v[e], v[e + 1], v[e], v[e + 1], inv_sqrt_d<D>(), inv_sqrt_d<D>());
}

// Row-major codes, blocks of at most 128 rows, one persistent launch.  For each block, thread
// 0 issues the tiled copies (d / 64 boxes of 64 columns, 128-byte swizzle: the 16-byte chunk c
// of row r sits at chunk c ^ (r & 7) of the row's 128 bytes) kRowBufs - 1 blocks ahead of the
// warps.  Thread t reads row t without bank conflicts, flips the signs by xor on the bf16 bits
// (exact, as multiplying by +-1), rotates the row in registers, and after the amax reduction
// writes the row's codes into its own slot of the first box (same swizzle); the CTA then
// stores the block's codes, contiguous rows in global memory, with coalesced stores.
template <int D, bool kRot>
__global__ void __launch_bounds__(kRowThreads, kRowCtasPerSm)
quant_rows_kernel(const __grid_constant__ CUtensorMap tmX, uint8_t* __restrict__ out,
                  float* __restrict__ scales, int N, int block_rows, int nblk, long long nsc,
                  const float* __restrict__ signs, int vec16, uint32_t* err) {
  constexpr int kBoxes = D / 64;
  constexpr uint32_t kBufBytes = kBoxes * kRowBoxBytes;
  constexpr int kChunks = D / 16;                     // 16-byte chunks of codes per row
  extern __shared__ uint8_t rows_smem_raw[];
  uint8_t* smem = rows_smem_raw + ((1024u - (smem_u32(rows_smem_raw) & 1023u)) & 1023u);
  // [kRowBufs blocks][sign masks: d / 2 words][mbarriers][4 warp maxima]
  uint32_t* s_sign = reinterpret_cast<uint32_t*>(smem + kRowBufs * kBufBytes);
  const uint32_t bars = smem_u32(s_sign + D / 2);
  float* s_amax = reinterpret_cast<float*>(s_sign + D / 2 + 2 * kRowBufs);
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int b) { return bars + 8u * (uint32_t)b; };
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (t == 0) {
    for (int b = 0; b < kRowBufs; ++b) mbar_init(bar(b), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
  }
  if (kRot && t < D / 2)   // bits 15 and 31 of word j flip the signs of columns 2j and 2j + 1
    s_sign[t] = (__ldg(signs + 2 * t) < 0.f ? 0x8000u : 0u) |
                (__ldg(signs + 2 * t + 1) < 0.f ? 0x80000000u : 0u);
  __syncthreads();
  auto issue = [&](long long id, int b) {
    const int bh = (int)(id / nblk);
    const int r0 = (int)(id % nblk) * block_rows;
    mbar_arrive_expect_tx(bar(b), (uint32_t)(kBoxes * block_rows * 128));
#pragma unroll
    for (int h = 0; h < kBoxes; ++h)
      tma_load_3d(sbase + (uint32_t)b * kBufBytes + h * kRowBoxBytes, &tmX, bar(b), 64 * h, r0,
                  bh);
  };
  if (t == 0)
    for (int k = 0; k < kRowBufs - 1; ++k)
      if (blockIdx.x + (long long)k * gridDim.x < nsc) issue(blockIdx.x + (long long)k * gridDim.x, k);
  int it = 0;
  for (long long id = blockIdx.x; id < nsc; id += gridDim.x, ++it) {
    const int b = it % kRowBufs;
    const long long ahead = id + (long long)(kRowBufs - 1) * gridDim.x;
    if (t == 0 && ahead < nsc) issue(ahead, (it + kRowBufs - 1) % kRowBufs);
    const bool ok = __syncthreads_and(mbar_wait(bar(b), (it / kRowBufs) & 1, nullptr, err,
                                                kSiteQuantLoad));
    if (!ok) {   // wait for the copies issued for the blocks ahead, then leave
      if (t == 0)
        for (int k = 1; k < kRowBufs; ++k)
          if (id + (long long)k * gridDim.x < nsc)
            mbar_wait(bar((it + k) % kRowBufs), ((it + k) / kRowBufs) & 1, nullptr, err,
                      kSiteQuantLoad);
      return;
    }
    const long long bh = id / nblk;
    const int blk = (int)(id % nblk);
    const int r0 = blk * block_rows;
    const int nrows = min(block_rows, N - r0);
    uint8_t* buf = smem + (uint32_t)b * kBufBytes;
    float v[D];
    if (t < nrows) {
#pragma unroll
      for (int h = 0; h < kBoxes; ++h)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(buf + h * kRowBoxBytes + t * 128 +
                                                          ((c ^ (t & 7)) << 4));
          uint32_t w[4] = {u.x, u.y, u.z, u.w};
          if constexpr (kRot) {
            const uint4 sg = *reinterpret_cast<const uint4*>(s_sign + h * 32 + c * 4);
            w[0] ^= sg.x;
            w[1] ^= sg.y;
            w[2] ^= sg.z;
            w[3] ^= sg.w;
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            v[h * 64 + c * 8 + 2 * i] = __uint_as_float(w[i] << 16);
            v[h * 64 + c * 8 + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
          }
        }
    } else {
#pragma unroll
      for (int e = 0; e < D; ++e) v[e] = 0.f;
    }
    if constexpr (kRot) hadamard_row<D>(v);
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < D; e += 2) m = max3f(m, fabsf(v[e]), fabsf(v[e + 1]));
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
    if (lane == 0) s_amax[warp] = m;
    __syncthreads();
    const float amax = fmaxf(fmaxf(s_amax[0], s_amax[1]), fmaxf(s_amax[2], s_amax[3]));
    const float inv = amax > 0.f ? kE4m3Max / amax : 1.f;
    if (t == 0) scales[bh * nblk + blk] = amax > 0.f ? amax / kE4m3Max : 1.f;
    if (t < nrows) {
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        float x[16];
#pragma unroll
        for (int j = 0; j < 16; j += 2)
          fmul2(x[j], x[j + 1], v[16 * c + j], v[16 * c + j + 1], inv, inv);
        const uint4 q = make_uint4(pack_e4m3x4(x[0], x[1], x[2], x[3]),
                                   pack_e4m3x4(x[4], x[5], x[6], x[7]),
                                   pack_e4m3x4(x[8], x[9], x[10], x[11]),
                                   pack_e4m3x4(x[12], x[13], x[14], x[15]));
        *reinterpret_cast<uint4*>(buf + t * 128 + ((c ^ (t & 7)) << 4)) = q;
      }
    }
    __syncthreads();
    uint8_t* dst = out + (bh * N + r0) * D;
    for (int q = t; q < nrows * kChunks; q += kRowThreads) {
      const int row = q / kChunks, c = q % kChunks;
      const uint4 val = *reinterpret_cast<const uint4*>(buf + row * 128 + ((c ^ (row & 7)) << 4));
      if (vec16) {
        *reinterpret_cast<uint4*>(dst + 16 * q) = val;
      } else {
        uint32_t* d4 = reinterpret_cast<uint32_t*>(dst + 16 * q);
        d4[0] = val.x;
        d4[1] = val.y;
        d4[2] = val.z;
        d4[3] = val.w;
      }
    }
    // the buffer and s_amax are free for the copy and reduction kRowBufs - 1 blocks on
    fence_proxy_async_smem();
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------- vt kernel
constexpr int kVtThreads = 128;
constexpr int kVtCluster = 8;                         // CTAs per head
constexpr int kVtBufs = 3;

// V transposed with one scale per head: codes [d][n_pad] of each head.  The head's keys are
// cut into sub-blocks of 128; CTA `rank` of the head's cluster takes sub-blocks rank,
// rank + 8, ....  Pass 1 streams them through a ring of kVtBufs buffers (one bulk copy each)
// and takes the largest |bf16| bit pattern (the largest magnitude, for finite values); the
// eight CTAs then write their maxima into every CTA's shared memory and meet at a cluster
// barrier.  Pass 2 streams the same sub-blocks again -- the copies are issued during pass 1
// and the cluster's 1 MB or so of a head is still in L2 -- and thread (p, g) converts the
// column pair p over rows [g 128 / G, (g + 1) 128 / G) to codes, 16 keys per 16-byte chunk,
// staged as the tile [d][128 keys] (chunk c of column row j at chunk c ^ ((j + j / 8) & 7),
// conflict-free both ways), then stored with coalesced 16-byte stores.  Keys in [N, n_pad)
// get code 0.
template <int D>
__global__ void __launch_bounds__(kVtThreads, 2)
quant_vt_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ out,
                float* __restrict__ scales, int N, int n_pad, uint32_t* err) {
  constexpr uint32_t kBufBytes = 128 * D * 2;
  constexpr int kPairs = D / 2;                       // column pairs
  constexpr int kGroups = kVtThreads / kPairs;        // row groups: 2 (d = 128) or 4 (d = 64)
  constexpr int kRowsPer = 128 / kGroups;
  extern __shared__ __align__(128) uint8_t vt_smem[];
  // [kVtBufs sub-blocks][stage: d x 128 bytes][8 cluster maxima][4 warp maxima][mbarriers]
  uint8_t* stage = vt_smem + kVtBufs * kBufBytes;
  uint32_t* slots = reinterpret_cast<uint32_t*>(stage + D * 128);
  uint32_t* s_max = slots + kVtCluster;
  const uint32_t bars = smem_u32(s_max + 4);
  auto bar = [&](int b) { return bars + 8u * (uint32_t)b; };
  const uint32_t ring = smem_u32(vt_smem);
  const int t = threadIdx.x, warp = t >> 5;
  // every CTA of the cluster is running once all have arrived here (waited on before the
  // first write into another CTA's shared memory)
  cluster_arrive_relaxed();
  const int rank = (int)cluster_ctarank();
  const long long bh = blockIdx.x / kVtCluster;
  const int nsub = (n_pad + 127) / 128;
  const int nmine = rank < nsub ? (nsub - 1 - rank) / kVtCluster + 1 : 0;
  const int last_live = (N - 1) / 128;
  const int nlive = rank <= last_live ? min(nmine, (last_live - rank) / kVtCluster + 1) : 0;
  const int nload = 2 * nlive;                        // pass 1, then pass 2, same order
  if (t == 0) {
    for (int b = 0; b < kVtBufs; ++b) mbar_init(bar(b), 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto sub_of = [&](int k) { return rank + kVtCluster * (k < nlive ? k : k - nlive); };
  auto issue = [&](int k) {
    const int r0 = sub_of(k) * 128;
    const uint32_t bytes = (uint32_t)min(128, N - r0) * D * 2;
    const int b = k % kVtBufs;
    mbar_arrive_expect_tx(bar(b), bytes);
    bulk_load(ring + (uint32_t)b * kBufBytes, x + (bh * N + r0) * D, bytes, bar(b));
  };
  if (t == 0)
    for (int k = 0; k < kVtBufs - 1 && k < nload; ++k) issue(k);
  bool ok = true;
  int k = 0;
  uint32_t mx = 0u;                                   // two 16-bit maxima of |bf16| bits
  for (; k < nlive; ++k) {
    if (t == 0 && k + kVtBufs - 1 < nload) issue(k + kVtBufs - 1);
    const int b = k % kVtBufs;
    ok = __syncthreads_and(mbar_wait(bar(b), (k / kVtBufs) & 1, nullptr, err, kSiteQuantVt));
    if (!ok) break;
    const int rows = min(128, N - sub_of(k) * 128);
    const uint4* src = reinterpret_cast<const uint4*>(vt_smem + (uint32_t)b * kBufBytes);
    for (int q = t; q < rows * D / 8; q += kVtThreads) {
      const uint4 u = src[q];
      mx = __vmaxu2(mx, u.x & 0x7fff7fffu);
      mx = __vmaxu2(mx, u.y & 0x7fff7fffu);
      mx = __vmaxu2(mx, u.z & 0x7fff7fffu);
      mx = __vmaxu2(mx, u.w & 0x7fff7fffu);
    }
    fence_proxy_async_smem();
    __syncthreads();
  }
  uint32_t m16 = max(mx & 0xffffu, mx >> 16);
  m16 = __reduce_max_sync(0xffffffffu, m16);
  if ((t & 31) == 0) s_max[warp] = m16;
  __syncthreads();
  const uint32_t cta_max = max(max(s_max[0], s_max[1]), max(s_max[2], s_max[3]));
  cluster_wait();
  if (t < kVtCluster) st_shared_cluster_u32(mapa_shared(smem_u32(slots + rank), (uint32_t)t), cta_max);
  cluster_arrive();
  cluster_wait();
  uint32_t head_max = 0u;
#pragma unroll
  for (int j = 0; j < kVtCluster; ++j) head_max = max(head_max, slots[j]);
  const float amax = __uint_as_float(head_max << 16);
  const float inv = amax > 0.f ? kE4m3Max / amax : 1.f;
  if (rank == 0 && t == 0) scales[bh] = amax > 0.f ? amax / kE4m3Max : 1.f;
  const int p = t % kPairs, g = t / kPairs;
  for (; ok && k < nload; ++k) {
    if (t == 0 && k + kVtBufs - 1 < nload) issue(k + kVtBufs - 1);
    const int b = k % kVtBufs;
    ok = __syncthreads_and(mbar_wait(bar(b), (k / kVtBufs) & 1, nullptr, err, kSiteQuantVt));
    if (!ok) break;
    const int s = sub_of(k);
    const int rows = min(128, N - s * 128);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(vt_smem + (uint32_t)b * kBufBytes);
#pragma unroll 1
    for (int c16 = 0; c16 < kRowsPer / 16; ++c16) {
      const int rbase = g * kRowsPer + 16 * c16;
      uint32_t w0[4], w1[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float a[4], e[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = rbase + 4 * j + i;
          const uint32_t w = r < rows ? src[r * kPairs + p] : 0u;
          fmul2(a[i], e[i], __uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u), inv, inv);
        }
        w0[j] = pack_e4m3x4(a[0], a[1], a[2], a[3]);
        w1[j] = pack_e4m3x4(e[0], e[1], e[2], e[3]);
      }
      const int c = rbase / 16;
      const int j0 = 2 * p, j1 = 2 * p + 1;
      *reinterpret_cast<uint4*>(stage + j0 * 128 + ((c ^ ((j0 + (j0 >> 3)) & 7)) << 4)) =
          make_uint4(w0[0], w0[1], w0[2], w0[3]);
      *reinterpret_cast<uint4*>(stage + j1 * 128 + ((c ^ ((j1 + (j1 >> 3)) & 7)) << 4)) =
          make_uint4(w1[0], w1[1], w1[2], w1[3]);
    }
    __syncthreads();
    uint8_t* dst = out + bh * D * (long long)n_pad + s * 128;
    for (int q = t; q < D * 8; q += kVtThreads) {
      const int j = q >> 3, c = q & 7;
      if (s * 128 + 16 * c < n_pad)
        *reinterpret_cast<uint4*>(dst + (long long)j * n_pad + 16 * c) =
            *reinterpret_cast<const uint4*>(stage + j * 128 + ((c ^ ((j + (j >> 3)) & 7)) << 4));
    }
    fence_proxy_async_smem();
    __syncthreads();
  }
  if (!ok) {   // wait for the copies still in flight, then leave
    if (t == 0)
      for (int j = k + 1; j < nload && j < k + kVtBufs; ++j)
        mbar_wait(bar(j % kVtBufs), (j / kVtBufs) & 1, nullptr, err, kSiteQuantVt);
    return;
  }
  // sub-blocks wholly past N (when n_pad reaches past the last one with keys): zeros
  for (int i = nlive; i < nmine; ++i) {
    const int s = rank + kVtCluster * i;
    uint8_t* dst = out + bh * D * (long long)n_pad + s * 128;
    for (int q = t; q < D * 8; q += kVtThreads) {
      const int j = q >> 3, c = q & 7;
      if (s * 128 + 16 * c < n_pad)
        *reinterpret_cast<uint4*>(dst + (long long)j * n_pad + 16 * c) = make_uint4(0, 0, 0, 0);
    }
  }
}

// Pass 3: scales from the block maxima.
__global__ void quant_finalize_kernel(float* scales, long long n) {
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float amax = __uint_as_float(reinterpret_cast<unsigned int*>(scales)[i]);
  scales[i] = amax > 0.f ? amax / kE4m3Max : 1.f;
}

template <int D>
int launch_quant(const CUtensorMap* tmx, const void* x, void* out, float* scales, int B, int H,
                 int N, int block_rows, int transpose, int n_pad, const float* signs,
                 uint32_t* err, int num_sms, cudaStream_t stream) {
  const int nblk = (N + block_rows - 1) / block_rows;
  const long long nsc = (long long)B * H * nblk;
  const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  const uintptr_t oa = reinterpret_cast<uintptr_t>(out);
  if (!transpose && block_rows <= 128 && tmx != nullptr) {
    constexpr int kSmem = kRowBufs * kRowBoxBytes * (D / 64) + D / 2 * 4 + 8 * kRowBufs + 16 + 1024;
    const auto kern = signs != nullptr ? quant_rows_kernel<D, true> : quant_rows_kernel<D, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
        cudaSuccess)
      return -4;
    const long long grid = std::min<long long>(nsc, (long long)num_sms * kRowCtasPerSm);
    kern<<<(unsigned)grid, kRowThreads, kSmem, stream>>>(
        *tmx, reinterpret_cast<uint8_t*>(out), scales, N, block_rows, nblk, nsc, signs,
        (oa & 15u) == 0 ? 1 : 0, err);
    return cudaGetLastError() == cudaSuccess ? 0 : -4;
  }
  if (transpose && signs == nullptr && nblk == 1 && n_pad % 16 == 0 && (oa & 15u) == 0) {
    constexpr int kSmem = kVtBufs * 128 * D * 2 + D * 128 + 4 * (kVtCluster + 4) + 8 * kVtBufs;
    if (cudaFuncSetAttribute(quant_vt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmem) != cudaSuccess)
      return -4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((long long)B * H * kVtCluster));
    cfg.blockDim = dim3(kVtThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kVtCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, quant_vt_kernel<D>, xb, reinterpret_cast<uint8_t*>(out), scales,
                           N, n_pad, err) != cudaSuccess)
      return -4;
    return cudaGetLastError() == cudaSuccess ? 0 : -4;
  }
  const int nchunk_in = (N + kChunkRows - 1) / kChunkRows;
  const int rows_out = transpose ? (n_pad > N ? n_pad : N) : N;
  const int nchunk_out = (rows_out + kChunkRows - 1) / kChunkRows;
  auto* bits = reinterpret_cast<unsigned int*>(scales);
  // transposed stores: 2 = staged 16-byte runs, 1 = 8-byte stores, 0 = byte stores
  const int wide = !transpose ? 0
                   : (n_pad % 16 == 0 && (oa & 15u) == 0) ? 2
                   : (n_pad % 8 == 0 && (oa & 7u) == 0)   ? 1
                                                          : 0;
  if (cudaMemsetAsync(scales, 0, (size_t)nsc * sizeof(float), stream) != cudaSuccess) return -4;
  quant_amax_kernel<D><<<(unsigned)((long long)B * H * nchunk_in), kQuantThreads, 0, stream>>>(
      xb, bits, N, block_rows, nblk, nchunk_in, signs);
  quant_codes_kernel<D><<<(unsigned)((long long)B * H * nchunk_out), kQuantThreads, 0, stream>>>(
      xb, reinterpret_cast<uint8_t*>(out), bits, N, block_rows, nblk, nchunk_out, transpose,
      n_pad, wide, signs);
  quant_finalize_kernel<<<(unsigned)((nsc + 255) / 256), 256, 0, stream>>>(scales, nsc);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace

int launch_quantize_e4m3(const CUtensorMap* tmx, const void* x, void* out, float* scales, int B,
                         int H, int N, int d, int block_rows, int transpose, int n_pad,
                         const float* signs, uint32_t* err, int num_sms, cudaStream_t stream) {
  if ((long long)B * H * N <= 0) return 0;
  if (d == 128) return launch_quant<128>(tmx, x, out, scales, B, H, N, block_rows, transpose,
                                         n_pad, signs, err, num_sms, stream);
  if (d == 64) return launch_quant<64>(tmx, x, out, scales, B, H, N, block_rows, transpose,
                                       n_pad, signs, err, num_sms, stream);
  return -2;
}

}  // namespace attn
