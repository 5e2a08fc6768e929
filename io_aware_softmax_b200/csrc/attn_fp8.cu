// FP8 (E4M3) inputs for the fused attention: block quantization with optional incoherent
// processing ("FlashAttention 논문 분석: IO-Aware Exact Attention", section "FP8 지원과 정확도
// 유지"): every block of `block_rows` rows of one (batch, head) gets its own scale
// (amax / 448, 448 being the largest finite E4M3 value), and Q and K may first be multiplied
// by the orthogonal matrix diag(signs) H / sqrt(d) (H the Sylvester Hadamard matrix), which
// leaves Q K^T unchanged and spreads outlier columns over all of d.
//
// One CTA per (batch, head, block), one warp per row: lane l holds columns
// [l d/32, (l + 1) d/32); the Hadamard butterflies run in registers and across lanes with
// shuffles.  Pass 1 reduces the block's amax, pass 2 rounds x * (448 / amax) to E4M3 (round
// to nearest even, saturating) and writes codes row-major, or transposed ([d][n_pad] per
// head, the K-major layout of V for the P V product) with the padding columns zeroed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "attn_internal.h"

namespace attn {

namespace {

constexpr int kQuantThreads = 256;
constexpr float kE4m3Max = 448.0f;

template <int D>
__device__ __forceinline__ void load_row(const __nv_bfloat16* __restrict__ x, long long row,
                                         const float* __restrict__ signs, float (&v)[D / 32]) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16* src = x + row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = __bfloat162float(src[e]);
  if (signs != nullptr) {
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] *= __ldg(signs + lane * E + e);
    // Walsh-Hadamard butterflies: pairs (i, i ^ s) for s = 1, 2, ..., D / 2; the low index
    // gets a + b, the high one a - b.  Strides below E stay in the lane.
#pragma unroll
    for (int s = 1; s < E; s <<= 1)
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (!(e & s)) {
          const float a = v[e], b = v[e + s];
          v[e] = a + b;
          v[e + s] = a - b;
        }
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
      const bool high = lane & s;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float o = __shfl_xor_sync(0xffffffffu, v[e], s);
        v[e] = high ? (o - v[e]) : (v[e] + o);
      }
    }
    const float norm = rsqrtf((float)D);
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] *= norm;
  }
}

template <int D>
__global__ void __launch_bounds__(kQuantThreads)
attn_quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ out,
                          float* __restrict__ scales, int H, int N, int block_rows, int nblk,
                          int transpose, int n_pad, const float* __restrict__ signs) {
  constexpr int E = D / 32;
  __shared__ unsigned int s_amax;
  const int bh = blockIdx.x / nblk, blk = blockIdx.x % nblk;
  const int r0 = blk * block_rows, r1 = min(N, r0 + block_rows);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kQuantThreads / 32;
  if (threadIdx.x == 0) s_amax = 0u;
  __syncthreads();
  float amax = 0.f;
  for (int r = r0 + warp; r < r1; r += nwarps) {
    float v[E];
    load_row<D>(x, (long long)bh * N + r, signs, v);
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(v[e]));
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
  if (lane == 0) atomicMax(&s_amax, __float_as_uint(amax));   // non-negative: order of bits
  __syncthreads();
  amax = __uint_as_float(s_amax);
  const float inv = amax > 0.f ? kE4m3Max / amax : 1.f;
  if (threadIdx.x == 0) scales[(long long)bh * nblk + blk] = amax > 0.f ? amax / kE4m3Max : 1.f;
  for (int r = r0 + warp; r < r1; r += nwarps) {
    float v[E];
    load_row<D>(x, (long long)bh * N + r, signs, v);
    uint8_t c[E];
#pragma unroll
    for (int e = 0; e < E; ++e)
      c[e] = (uint8_t)__nv_cvt_float_to_fp8(v[e] * inv, __NV_SATFINITE, __NV_E4M3);
    if (!transpose) {
      uint8_t* dst = out + ((long long)bh * N + r) * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) dst[e] = c[e];
    } else {
      uint8_t* dst = out + (long long)bh * D * n_pad + r;
#pragma unroll
      for (int e = 0; e < E; ++e) dst[(long long)(lane * E + e) * n_pad] = c[e];
    }
  }
  // the padding columns [N, n_pad) of a transposed output hold zero codes
  if (transpose && blk == nblk - 1 && n_pad > N) {
    uint8_t* base = out + (long long)bh * D * n_pad;
    const int w = n_pad - N;
    for (int i = threadIdx.x; i < D * w; i += kQuantThreads)
      base[(long long)(i / w) * n_pad + N + i % w] = 0;
  }
}

}  // namespace

int launch_quantize_e4m3(const void* x, void* out, float* scales, int B, int H, int N, int d,
                         int block_rows, int transpose, int n_pad, const float* signs,
                         cudaStream_t stream) {
  const int nblk = (N + block_rows - 1) / block_rows;
  const long long grid = (long long)B * H * nblk;
  if (grid <= 0) return 0;
  const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  auto* ob = reinterpret_cast<uint8_t*>(out);
  if (d == 128)
    attn_quantize_e4m3_kernel<128><<<(unsigned)grid, kQuantThreads, 0, stream>>>(
        xb, ob, scales, H, N, block_rows, nblk, transpose, n_pad, signs);
  else if (d == 64)
    attn_quantize_e4m3_kernel<64><<<(unsigned)grid, kQuantThreads, 0, stream>>>(
        xb, ob, scales, H, N, block_rows, nblk, transpose, n_pad, signs);
  else
    return -2;
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace attn
