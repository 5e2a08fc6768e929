// Mask hooks of the fused attention kernels.
//
// Every supported mask gives each query row q one contiguous interval of visible keys
// [lo(q), hi(q)], and both ends are non-decreasing in q:
//   none              [0, Nk-1]
//   causal            [0, q]                       key <= query, diagonal visible
//   sliding + causal  [max(0, q - window), q]      |q - kv| <= window and kv <= q
//   document + causal [start of q's document, q]   same packed sequence and kv <= q
//   sliding           [max(0, q - window), q + window]   |q - kv| <= window, no causality
// (score_mod/mask hooks of "PyTorch FlexAttention 도입 분석", section 2, with the
// sliding_window_mod example; document boundaries as the cu_seqlens of "3.7 어텐션 II",
// section 3.7.6; causal masking as in "Attention 최적화가 어려운 이유", "Attention의 계산
// 흐름").  The interval form makes the per-element test two compares and lets a whole
// 128x128 tile be classified empty / partial / full in O(1) (the BlockMask early-out of the
// FlexAttention page).
#pragma once

#include <cstdint>

namespace attn {

enum MaskKind : int {
  kMaskNone = 0, kMaskCausal = 1, kMaskSlidingCausal = 2, kMaskDocCausal = 3, kMaskSliding = 4
};
enum TileClass : uint8_t { kTileEmpty = 0, kTilePartial = 1, kTileFull = 2 };

struct MaskParams {
  int kind;
  int window;
  const int* doc_offsets;   // device int32 [num_docs + 1]: 0 = o_0 <= o_1 <= ... <= o_n = Nk
  int num_docs;
  int Nq;
  int Nk;
};

// Start of the document holding position q: the largest o_i (i < num_docs) with o_i <= q.
__device__ __forceinline__ int doc_start(const int* __restrict__ offs, int num_docs, int q) {
  int lo = 0, hi = num_docs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(offs + mid) <= q) lo = mid; else hi = mid - 1;
  }
  return __ldg(offs + lo);
}

__device__ __forceinline__ void row_interval(const MaskParams& m, int q, int& lo, int& hi) {
  const int last = m.Nk - 1;
  switch (m.kind) {
    case kMaskCausal:
      lo = 0;
      hi = min(q, last);
      break;
    case kMaskSlidingCausal:
      lo = max(0, q - m.window);
      hi = min(q, last);
      break;
    case kMaskDocCausal:
      lo = doc_start(m.doc_offsets, m.num_docs, q);
      hi = min(q, last);
      break;
    case kMaskSliding:
      lo = max(0, q - m.window);
      hi = (int)min((long long)q + m.window, (long long)last);
      break;
    default:
      lo = 0;
      hi = last;
      break;
  }
}

// Class of the tile rows [q0, q1) x keys [k0, k1) (both already clipped to Nq / Nk),
// counting only the pairs inside it.
__device__ __forceinline__ int classify_tile(const MaskParams& m, int q0, int q1, int k0, int k1) {
  int lo_f, hi_f, lo_l, hi_l;
  row_interval(m, q0, lo_f, hi_f);
  row_interval(m, q1 - 1, lo_l, hi_l);
  if (lo_l <= k0 && k1 - 1 <= hi_f) return kTileFull;
  // The row with the smallest lo whose interval reaches k0 is the first row with hi >= k0.
  const int first = (m.kind == kMaskNone) ? q0
                    : (m.kind == kMaskSliding) ? (int)max((long long)q0, (long long)k0 - m.window)
                                               : max(q0, k0);
  if (first >= q1) return kTileEmpty;
  int lo, hi;
  row_interval(m, first, lo, hi);
  return (lo <= k1 - 1 && hi >= k0 && lo <= hi) ? kTilePartial : kTileEmpty;
}

}  // namespace attn
