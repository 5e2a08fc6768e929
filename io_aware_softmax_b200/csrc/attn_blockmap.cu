// Block-sparsity map of a mask at 128x128 granularity: for every (batch, query tile, key
// tile) whether no pair, some pairs or all pairs of the tile are visible.  This is the
// BlockMask precomputation of "PyTorch FlexAttention 도입 분석" (section 2: tiles that need
// no work are skipped, bringing O(N^2) towards O(N) for causal, windowed and packed-document
// masks).  The prefill kernel evaluates the same classify_tile() inline for its own tiles;
// this kernel materialises the map for callers that want it.
#include <cuda_runtime.h>

#include "attn_internal.h"
#include "mask.cuh"

namespace attn {

namespace {

__global__ void attn_blockmap_kernel(const MaskParams m, int B, int nqt, int nkt, uint8_t* map) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)nqt * nkt) return;
  const int i = (int)(idx / nkt);
  const int j = (int)(idx % nkt);
  const int q0 = i * 128, q1 = min(q0 + 128, m.Nq);
  const int k0 = j * 128, k1 = min(k0 + 128, m.Nk);
  const uint8_t cls = (uint8_t)classify_tile(m, q0, q1, k0, k1);
  for (int b = 0; b < B; ++b) map[((long long)b * nqt + i) * nkt + j] = cls;
}

}  // namespace

int launch_blockmap(const MaskParams& m, int B, int Nq, int Nk, uint8_t* map,
                    cudaStream_t stream) {
  const int nqt = (Nq + 127) / 128;
  const int nkt = (Nk + 127) / 128;
  const long long n = (long long)nqt * nkt;
  if (n == 0 || B == 0) return 0;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  attn_blockmap_kernel<<<blocks, 256, 0, stream>>>(m, B, nqt, nkt, map);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace attn
