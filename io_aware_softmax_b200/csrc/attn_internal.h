// Declarations shared by the kernels' launch wrappers and the C-ABI entry points.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "mask.cuh"

namespace attn {

// Cost-ordered scheduling of the prefill (FwdParams::sched): at most kSchedUnits work units
// in all (their sort keys fill 16 KB of the K/V ring before it is used) and kSchedMax per CTA.
constexpr int kSchedUnits = 4096;
constexpr int kSchedMax = 63;

struct FwdParams {
  void* o;            // bf16 [B, Hq, Nq, d]
  float* lse;         // fp32 [B, Hq, Nq]
  int B, Hq, Hkv, Nq, Nk;
  int G;              // Hq / Hkv
  int num_pairs;      // work units per (b, h) [adjacent tiles: ceil(Nq / 256)] or per
                      // (b, head pair) [head pairs: ceil(Nq / 128)]
  int head_pairs;     // 1: a CTA's two query tiles are query heads 2m, 2m + 1 at the same rows
  int sched;          // 1: units dealt by cost (sorted, snake) instead of in index order
  int num_sms;        // persistent grid size (SMs of the device)
  float kscale;       // scale * log2(e)
  float softcap;      // > 0: soft-cap enabled
  float cap_scale;    // scale / softcap
  float cap_log2;     // softcap * log2(e)
  // Soft-cap on the FMA pipe: cap_log2 * tanh(s cap_scale) = s * sum_i cap_poly[i] s^(2i)
  // for raw scores |s| <= cap_fast_max (|s cap_scale| <= 1/2); cap_fast_max < 0 disables it
  float cap_poly[5];
  float cap_fast_max;
  // Units visit their K/V tiles last to first (ALiBi: the tiles nearest the diagonal hold
  // the row maxima, so O is hardly ever rescaled; other calls keep the ascending order,
  // which measured faster under a plain causal mask).
  int kv_reverse;
  MaskParams mask;
  const float* alibi; // fp32 [Hq] ALiBi slopes (natural-log units per key of distance) or null
  // FP8 (E4M3) inputs, null otherwise: per 128-row block scales of Q and K, per head of V
  const float* q_scales;  // fp32 [B, Hq, nqt]
  const float* k_scales;  // fp32 [B, Hkv, nkt]
  const float* v_scales;  // fp32 [B, Hkv]
  int nqt, nkt;           // ceil(Nq / 128), ceil(Nk / 128)
  uint32_t* err;      // device error word of the library (bits, first site)
};

struct DecParams {
  const void* q;      // bf16 [B, Hq, 1, d]
  float* o_part;      // fp32 [B, Hq, S, d]: each split normalised by its own sum
  float* lse_part;    // fp32 [B, Hq, S]: natural-log LSE of each split (-inf if empty)
  int B, Hq, Hkv, T, S;
  int num_items;      // B * Hkv * S
  float kscale;       // scale * log2(e)
  uint32_t* err;      // device error word of the library (bits, first site)
  // Paged, variable-length caches (null / 0 for one contiguous cache of T rows each):
  const int* block_table;   // int32 [B, max_pages]: physical page of each logical page
  const int* seq_lens;      // int32 [B]: cache rows of each sequence
  int page_size;            // rows per page (a multiple of the 64-row tile)
  int max_pages;            // pages per block-table row
};

struct BwdParams {
  void* dq;           // bf16 [B, Hq, Nq, d]  (written)
  void* dk;           // bf16 [B, Hkv, Nk, d] (written)
  void* dv;           // bf16 [B, Hkv, Nk, d] (written)
  const float* dvec;  // fp32 [B, Hq, Nq]: rowsum(dO * O)
  const float* l2;    // fp32 [B, Hq, Nq]: LSE * log2(e), +inf for rows without a key
  int B, Hq, Hkv, Nq, Nk;
  int G;              // Hq / Hkv
  float kscale;       // scale * log2(e)
  float scale;
  MaskParams mask;
  const float* alibi;  // fp32 [Hq] ALiBi slopes (natural-log units), or nullptr
  float cap_scale;    // soft-cap c > 0: scale / c (0: no cap)
  float cap_log2;     // c * log2(e)
  float cap_poly[5];  // the polynomial tanh, as FwdParams::cap_poly
  float cap_fast_max; // as FwdParams::cap_fast_max
  uint32_t* err;      // device error word of the library (bits, first site)
};

int launch_attn_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const FwdParams& p, int d, cudaStream_t stream);
int launch_fill_empty(void* o, float* lse, size_t rows, int d, cudaStream_t stream);
int launch_blockmap(const MaskParams& m, int B, int Nq, int Nk, uint8_t* map,
                    cudaStream_t stream);
int launch_decode_split(const CUtensorMap& tk, const CUtensorMap& tv, const DecParams& p,
                        int d, int G, int grid, cudaStream_t stream);
int decode_ctas_per_sm(int d, int G);
int launch_bwd_rowdot(const void* o, const void* dout, const float* lse, float* dvec, float* l2,
                      long long rows, int d, cudaStream_t stream);
int launch_attn_bwd(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                    const CUtensorMap& tv, const BwdParams& p, int d, cudaStream_t stream);
// tmx: tiled map of x (make_map_3d over [B H, N, d] with block_rows-row boxes) for
// row-major blocks of at most 128 rows, or nullptr.
int launch_quantize_e4m3(const CUtensorMap* tmx, const void* x, void* out, float* scales, int B,
                         int H, int N, int d, int block_rows, int transpose, int n_pad,
                         const float* signs, uint32_t* err, int num_sms, cudaStream_t stream);
int launch_merge(const float* o_part, const float* lse_part, void* o, float* lse, long long rows,
                 int S, int d, cudaStream_t stream);

}  // namespace attn
