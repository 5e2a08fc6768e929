// FP8 (E4M3) inputs for the fused attention: block quantization with optional incoherent
// processing ("FlashAttention 논문 분석: IO-Aware Exact Attention", section "FP8 지원과 정확도
// 유지"): every block of `block_rows` rows of one (batch, head) gets its own scale
// (amax / 448, 448 being the largest finite E4M3 value), and Q and K may first be multiplied
// by the orthogonal matrix diag(signs) H / sqrt(d) (H the Sylvester Hadamard matrix), which
// leaves Q K^T unchanged and spreads outlier columns over all of d.
//
// Row-major output with blocks of at most 128 rows: one launch, one CTA per block, the block
// brought in by one bulk copy and held in registers between its amax and its codes (read
// once).
// Larger blocks or a transposed output: three launches over chunks of 64 rows of one
// (batch, head), 256 threads each, a warp per 8 consecutive rows.  In both, lane l holds
// columns [l d/32, (l + 1) d/32) of a row and the Hadamard butterflies run in registers and
// across lanes with shuffles.  The chunked launches:
//   1. amax: each chunk reduces the |values| of every block it touches in shared memory and
//      folds them into `scales` (zeroed first) with one atomic max per block, as float bits;
//   2. quantize: x * (448 / amax) rounded to E4M3 (nearest even, saturating), written
//      row-major, or transposed ([d][n_pad] per head, the K-major layout of V for the P V
//      product; columns [N, n_pad) zero) -- staged in shared memory and written in 16-byte
//      runs of each column when n_pad allows, else 8 rows of one column per 8-byte store;
//   3. finalize: scales = amax / 448 (1 for an all-zero block).
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
  const float norm = rsqrtf((float)D);
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = __fmul_rn(v[e], norm);
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

// Row-major blocks of at most 128 rows in one pass.  A persistent grid of eight-warp CTAs
// walks the blocks; for each, one thread copies the whole block (contiguous rows) into shared
// memory with a single bulk copy, and the copies of the CTA's next blocks are issued before
// this one is processed (three buffers), so copies are always in flight while the warps
// compute.
// Warp w takes rows w, w + 8, ... of the block, rotates them and holds them in registers
// while the block's amax is reduced, then writes the codes from the same registers: the
// input is read once.
constexpr int kBlockThreads = 256;
constexpr int kBlockCtasPerSm = 2;
constexpr int kBlockBufs = 3;                         // 3 x 32 KB of buffers per CTA
constexpr uint32_t kSiteQuantLoad = 0x51u;

template <int D>
__global__ void __launch_bounds__(kBlockThreads, kBlockCtasPerSm)
quant_block_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ out,
                   float* __restrict__ scales, int N, int block_rows, int nblk, long long nsc,
                   const float* __restrict__ signs, uint32_t* err) {
  constexpr int E = D / 32;
  constexpr int kWarps = kBlockThreads / 32;
  constexpr int kRows = 128 / kWarps;                 // rows per warp, at most
  constexpr uint32_t kBufBytes = 128 * D * 2;
  extern __shared__ __align__(128) uint8_t qsmem[];   // kBlockBufs blocks of rows, then mbarriers
  __shared__ float s_amax[kWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbuf = smem_u32(qsmem);
  auto bar = [&](int b) { return sbuf + kBlockBufs * kBufBytes + 8u * (uint32_t)b; };
  if (threadIdx.x == 0) {
    for (int b = 0; b < kBlockBufs; ++b) mbar_init(bar(b), 1);
    fence_mbar_init();
  }
  __syncthreads();
  // the copy of block `id` into buffer `b` (issued by thread 0)
  auto issue = [&](long long id, int b) {
    const long long bh = id / nblk;
    const int r0 = (int)(id % nblk) * block_rows;
    const int r1 = min(N, r0 + block_rows);
    const uint32_t bytes = (uint32_t)(r1 - r0) * D * 2;
    mbar_arrive_expect_tx(bar(b), bytes);
    bulk_load(sbuf + (uint32_t)b * kBufBytes, x + (bh * N + r0) * D, bytes, bar(b));
  };
  // the CTA's k-th block is blockIdx.x + k * gridDim.x and goes to buffer k % kBlockBufs;
  // copies run kBlockBufs - 1 blocks ahead of the warps
  if (threadIdx.x == 0)
    for (int k = 0; k < kBlockBufs - 1; ++k)
      if (blockIdx.x + (long long)k * gridDim.x < nsc) issue(blockIdx.x + (long long)k * gridDim.x, k);
  int it = 0;
  for (long long id = blockIdx.x; id < nsc; id += gridDim.x, ++it) {
    const int b = it % kBlockBufs;
    // the buffer of the block kBlockBufs - 1 ahead was released by the barrier that ended the
    // previous iteration
    const long long ahead = id + (long long)(kBlockBufs - 1) * gridDim.x;
    if (threadIdx.x == 0 && ahead < nsc) issue(ahead, (it + kBlockBufs - 1) % kBlockBufs);
    // every thread waits; the CTA agrees on the outcome, and after a timeout thread 0 waits
    // for the copies it issued for the blocks ahead before the CTA leaves
    const bool ok = __syncthreads_and(mbar_wait(bar(b), (it / kBlockBufs) & 1, nullptr, err,
                                                kSiteQuantLoad));
    if (!ok) {
      if (threadIdx.x == 0)
        for (int k = 1; k < kBlockBufs; ++k)
          if (id + (long long)k * gridDim.x < nsc)
            mbar_wait(bar((it + k) % kBlockBufs), ((it + k) / kBlockBufs) & 1, nullptr, err,
                      kSiteQuantLoad);
      return;
    }
    const long long bh = id / nblk;
    const int blk = (int)(id % nblk);
    const int r0 = blk * block_rows, r1 = min(N, r0 + block_rows);
    const __nv_bfloat16* rows =
        reinterpret_cast<const __nv_bfloat16*>(qsmem + (uint32_t)b * kBufBytes);
    float v[kRows][E];
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int r = warp + i * kWarps;
      if (r0 + r < r1) {
        bf16_lane_values<D>(rows + r * D + lane * E, v[i]);
        if (signs != nullptr) rotate_row<D>(signs, v[i]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) v[i][e] = 0.f;
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < kRows; ++i)
#pragma unroll
      for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(v[i][e]));   // rows past r1 are 0
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
    if (lane == 0) s_amax[warp] = amax;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kWarps; ++w) amax = fmaxf(amax, s_amax[w]);
    const float inv = amax > 0.f ? kE4m3Max / amax : 1.f;
    if (threadIdx.x == 0) scales[bh * nblk + blk] = amax > 0.f ? amax / kE4m3Max : 1.f;
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int r = r0 + warp + i * kWarps;
      if (r >= r1) break;
      uint32_t c = 0;
#pragma unroll
      for (int e = 0; e < E; ++e)
        c |= (uint32_t)__nv_cvt_float_to_fp8(v[i][e] * inv, __NV_SATFINITE, __NV_E4M3)
             << (8 * e);
      uint8_t* dst = out + (bh * N + r) * D + lane * E;
      if constexpr (E == 4)
        *reinterpret_cast<uint32_t*>(dst) = c;
      else
        *reinterpret_cast<uint16_t*>(dst) = (uint16_t)c;
    }
    // buffer b and s_amax are free for the copy and reduction two iterations on
    __syncthreads();
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
int launch_quant(const void* x, void* out, float* scales, int B, int H, int N, int block_rows,
                 int transpose, int n_pad, const float* signs, uint32_t* err, int num_sms,
                 cudaStream_t stream) {
  const int nblk = (N + block_rows - 1) / block_rows;
  const long long nsc = (long long)B * H * nblk;
  const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  if (!transpose && block_rows <= 128) {
    constexpr int kSmem = kBlockBufs * 128 * D * 2 + 8 * kBlockBufs;
    if (cudaFuncSetAttribute(quant_block_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmem) != cudaSuccess)
      return -4;
    const long long grid = std::min<long long>(nsc, (long long)num_sms * kBlockCtasPerSm);
    quant_block_kernel<D><<<(unsigned)grid, kBlockThreads, kSmem, stream>>>(
        xb, reinterpret_cast<uint8_t*>(out), scales, N, block_rows, nblk, nsc, signs, err);
    return cudaGetLastError() == cudaSuccess ? 0 : -4;
  }
  const int nchunk_in = (N + kChunkRows - 1) / kChunkRows;
  const int rows_out = transpose ? (n_pad > N ? n_pad : N) : N;
  const int nchunk_out = (rows_out + kChunkRows - 1) / kChunkRows;
  auto* bits = reinterpret_cast<unsigned int*>(scales);
  // transposed stores: 2 = staged 16-byte runs, 1 = 8-byte stores, 0 = byte stores
  const uintptr_t oa = reinterpret_cast<uintptr_t>(out);
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

int launch_quantize_e4m3(const void* x, void* out, float* scales, int B, int H, int N, int d,
                         int block_rows, int transpose, int n_pad, const float* signs,
                         uint32_t* err, int num_sms, cudaStream_t stream) {
  if ((long long)B * H * N <= 0) return 0;
  if (d == 128) return launch_quant<128>(x, out, scales, B, H, N, block_rows, transpose, n_pad,
                                         signs, err, num_sms, stream);
  if (d == 64) return launch_quant<64>(x, out, scales, B, H, N, block_rows, transpose, n_pad,
                                       signs, err, num_sms, stream);
  return -2;
}

}  // namespace attn
