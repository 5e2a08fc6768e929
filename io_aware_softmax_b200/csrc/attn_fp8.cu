// FP8 (E4M3) inputs for the fused attention: block quantization with optional incoherent
// processing ("FlashAttention 논문 분석: IO-Aware Exact Attention", section "FP8 지원과 정확도
// 유지"): every block of `block_rows` rows of one (batch, head) gets its own scale
// (amax / 448, 448 being the largest finite E4M3 value), and Q and K may first be multiplied
// by the orthogonal matrix diag(signs) H / sqrt(d) (H the Sylvester Hadamard matrix), which
// leaves Q K^T unchanged and spreads outlier columns over all of d.
//
// Row-major output with blocks of at most 128 rows: one launch, one CTA per block, the
// block held in registers between its amax and its codes (read once).
// Larger blocks or a transposed output: three launches over chunks of 64 rows of one
// (batch, head), 256 threads each, a warp per 8 consecutive rows.  In both, lane l holds
// columns [l d/32, (l + 1) d/32) of a row and the Hadamard butterflies run in registers and
// across lanes with shuffles.  The chunked launches:
//   1. amax: each chunk reduces the |values| of every block it touches in shared memory and
//      folds them into `scales` (zeroed first) with one atomic max per block, as float bits;
//   2. quantize: x * (448 / amax) rounded to E4M3 (nearest even, saturating), written
//      row-major, or transposed ([d][n_pad] per head, the K-major layout of V for the P V
//      product; columns [N, n_pad) zero) -- 8 rows of one column per 8-byte store;
//   3. finalize: scales = amax / 448 (1 for an all-zero block).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "attn_internal.h"

namespace attn {

namespace {

constexpr int kQuantThreads = 256;
constexpr int kChunkRows = 64;
constexpr int kRowsPerWarp = kChunkRows / (kQuantThreads / 32);   // 8
constexpr float kE4m3Max = 448.0f;

// This lane's d/32 values of row `row` (zeros past the last row), rotated when signs != 0.
template <int D>
__device__ __forceinline__ void load_row(const __nv_bfloat16* __restrict__ x, long long row,
                                         bool valid, const float* __restrict__ signs,
                                         float (&v)[D / 32]) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  if (valid) {
    const __nv_bfloat16* src = x + row * D + lane * E;
    if constexpr (E == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(src);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
      v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    } else {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src));
      v[0] = a.x; v[1] = a.y;
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = 0.f;
  }
  if (signs != nullptr) {
    // explicitly rounded operations: both passes must produce the same bits (no FMA
    // contraction that could differ between the two kernels)
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
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
      const bool high = lane & s;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float o = __shfl_xor_sync(0xffffffffu, v[e], s);
        v[e] = high ? __fsub_rn(o, v[e]) : __fadd_rn(v[e], o);
      }
    }
    const float norm = rsqrtf((float)D);
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = __fmul_rn(v[e], norm);
  }
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
  if (w0 >= rows) return;
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

// Row-major blocks of at most 128 rows in one pass: one CTA per block, warp w holding rows
// w, w + 8, ... of it.  Every row of the block is loaded (and rotated) into registers before
// any is used -- 16 independent loads in flight per warp -- then the block's amax is reduced
// across the CTA and the codes are written from the same registers: the input is read once.
template <int D>
__global__ void __launch_bounds__(kQuantThreads)
quant_block_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ out,
                   float* __restrict__ scales, int N, int block_rows, int nblk,
                   const float* __restrict__ signs) {
  constexpr int E = D / 32;
  constexpr int kWarps = kQuantThreads / 32;
  constexpr int kRows = 128 / kWarps;                 // rows per warp, at most
  __shared__ float s_amax[kWarps];
  const int bh = blockIdx.x / nblk, blk = blockIdx.x % nblk;
  const int r0 = blk * block_rows, r1 = min(N, r0 + block_rows);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float v[kRows][E];
#pragma unroll
  for (int i = 0; i < kRows; ++i) {
    const int r = r0 + warp + i * kWarps;
    load_row<D>(x, (long long)bh * N + r, r < r1, signs, v[i]);
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
  if (threadIdx.x == 0) scales[(long long)bh * nblk + blk] = amax > 0.f ? amax / kE4m3Max : 1.f;
#pragma unroll
  for (int i = 0; i < kRows; ++i) {
    const int r = r0 + warp + i * kWarps;
    if (r >= r1) break;
    uint32_t c = 0;
#pragma unroll
    for (int e = 0; e < E; ++e)
      c |= (uint32_t)__nv_cvt_float_to_fp8(v[i][e] * inv, __NV_SATFINITE, __NV_E4M3) << (8 * e);
    uint8_t* dst = out + ((long long)bh * N + r) * D + lane * E;
    if constexpr (E == 4)
      *reinterpret_cast<uint32_t*>(dst) = c;
    else
      *reinterpret_cast<uint16_t*>(dst) = (uint16_t)c;
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
                 int transpose, int n_pad, const float* signs, cudaStream_t stream) {
  const int nblk = (N + block_rows - 1) / block_rows;
  const long long nsc = (long long)B * H * nblk;
  const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  if (!transpose && block_rows <= 128) {
    quant_block_kernel<D><<<(unsigned)nsc, kQuantThreads, 0, stream>>>(
        xb, reinterpret_cast<uint8_t*>(out), scales, N, block_rows, nblk, signs);
    return cudaGetLastError() == cudaSuccess ? 0 : -4;
  }
  const int nchunk_in = (N + kChunkRows - 1) / kChunkRows;
  const int rows_out = transpose ? (n_pad > N ? n_pad : N) : N;
  const int nchunk_out = (rows_out + kChunkRows - 1) / kChunkRows;
  auto* bits = reinterpret_cast<unsigned int*>(scales);
  const int wide = transpose && (n_pad % 8 == 0) &&
                   (reinterpret_cast<uintptr_t>(out) & 7u) == 0;
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
                         cudaStream_t stream) {
  if ((long long)B * H * N <= 0) return 0;
  if (d == 128) return launch_quant<128>(x, out, scales, B, H, N, block_rows, transpose, n_pad,
                                         signs, stream);
  if (d == 64) return launch_quant<64>(x, out, scales, B, H, N, block_rows, transpose, n_pad,
                                       signs, stream);
  return -2;
}

}  // namespace attn
