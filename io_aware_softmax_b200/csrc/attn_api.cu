// C-ABI entry points: argument validation, TMA descriptor construction and launches.
// Nothing here allocates device memory or synchronises (except attn_get_device_status).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <algorithm>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "attn_internal.h"
#include "sm100_ptx.cuh"
#include "tanh_poly.cuh"

namespace attn {

// The library's device error word: [0] = error bits, [1] = first failing wait site,
// [2..3] = limit of the kernels' pipeline waits in ns (64-bit; 0: the built-in 0.5 s).
__device__ __align__(8) uint32_t g_error[4] = {0u, 0u, 0u, 0u};

namespace {

constexpr float kLog2e = 1.4426950408889634f;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 3-D tensor map of bytes over [z, rows, inner] (inner = `extent` valid bytes of each
// `stride`-byte row) with a (128 x box_rows x 1) box and 128-byte swizzle; bytes past the
// extent read as zero.
bool make_map_3d_u8(CUtensorMap* map, const void* ptr, long long extent, long long stride,
                    long long rows, long long z, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)extent, (cuuint64_t)rows, (cuuint64_t)z};
  cuuint64_t strides[2] = {(cuuint64_t)stride, (cuuint64_t)stride * (cuuint64_t)rows};
  cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D bf16 tensor map over [z, rows, d] (d innermost) with a (64 x box_rows x 1) box and
// 128-byte swizzle: one box fills `box_rows` rows of 128 bytes in shared memory.
bool make_map_3d(CUtensorMap* map, const void* ptr, int d, long long rows, long long z,
                 int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)z};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * (cuuint64_t)rows};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The soft-cap's polynomial tanh in the raw score s: cap_log2 tanh(s cap_scale) =
// s sum_i b_i s^(2i) with b_i = cap_log2 a_i cap_scale^(2i + 1), for |s cap_scale| <= 1/2
// (fast_max = 1 / (2 cap_scale) in raw units).  The kernels take it only when every b_i is a
// normal float (no term flushed to zero); otherwise fast_max = -1 turns it off.
void soft_cap_poly(float cap_scale, float cap_log2, float (&poly)[kTanhPolyTerms],
                   float& fast_max) {
  // The leading coefficient is positive, so a masked score (-inf) comes out of the
  // polynomial as -inf: the kernels need no other mask on the polynomial path.
  static_assert(kTanhPoly[kTanhPolyTerms - 1] > 0.f, "leading coefficient");
  fast_max = -1.f;
  for (int i = 0; i < kTanhPolyTerms; ++i) poly[i] = 0.f;
  if (!(cap_scale > 0.f)) return;
  bool normal = true;
  double cs_pow = (double)cap_scale;
  for (int i = 0; i < kTanhPolyTerms; ++i) {
    poly[i] = (float)((double)kTanhPoly[i] * (double)cap_log2 * cs_pow);
    normal = normal && std::isnormal(poly[i]);
    cs_pow *= (double)cap_scale * (double)cap_scale;
  }
  if (normal) fast_max = kTanhPolyMaxY / cap_scale;
}

int check_mask(int mask_kind, int window, const int* doc_offsets, int num_docs, int Nq, int Nk) {
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_SLIDING) return ATTN_ERR_INVALID_ARG;
  if (mask_kind != ATTN_MASK_NONE && Nq != Nk) return ATTN_ERR_UNSUPPORTED;
  if ((mask_kind == ATTN_MASK_SLIDING_CAUSAL || mask_kind == ATTN_MASK_SLIDING) && window < 0)
    return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_DOCUMENT_CAUSAL) {
    if (doc_offsets == nullptr || num_docs < 1) return ATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(doc_offsets) & 3u) return ATTN_ERR_MISALIGNED;
  }
  return ATTN_OK;
}

MaskParams mask_params(int mask_kind, int window, const int* doc_offsets, int num_docs, int Nq,
                       int Nk) {
  MaskParams m;
  m.kind = mask_kind;
  m.window = window;
  m.doc_offsets = doc_offsets;
  m.num_docs = num_docs;
  m.Nq = Nq;
  m.Nk = Nk;
  return m;
}

int sm_count(int device) {
  static int cached[64] = {0};
  if (device >= 0 && device < 64 && cached[device] > 0) return cached[device];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n < 1)
    n = 148;
  if (device >= 0 && device < 64) cached[device] = n;
  return n;
}

// Device address of g_error on the current device (looked up once per device).
uint32_t* error_word_ptr(int device) {
  static std::mutex mu;
  static uint32_t* cache[64] = {};
  if (device < 0 || device >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[device] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_error) != cudaSuccess) return nullptr;
    cache[device] = reinterpret_cast<uint32_t*>(ptr);
  }
  return cache[device];
}

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return dev;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" int attn_version(void) { return 100; }

extern "C" const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ATTN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

extern "C" int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Nq, int Nk, int d, float scale, int mask_kind,
                        int window, float softcap, const int* doc_offsets, int num_docs,
                        cudaStream_t stream) {
  return attn_fwd_alibi(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, mask_kind, window, softcap,
                        doc_offsets, num_docs, nullptr, stream);
}

extern "C" int attn_fwd_alibi(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                              int mask_kind, int window, float softcap, const int* doc_offsets,
                              int num_docs, const float* alibi_slopes, cudaStream_t stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Hkv == 0 && Hq > 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv > 0 && Hq % Hkv != 0) return ATTN_ERR_UNSUPPORTED;
  int st = check_mask(mask_kind, window, doc_offsets, num_docs, Nq, Nk);
  if (st != ATTN_OK) return st;
  if (std::isnan(scale) || std::isnan(softcap)) return ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(alibi_slopes) & 3u) return ATTN_ERR_MISALIGNED;
  if (alibi_slopes != nullptr && softcap > 0.f) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || Hq == 0 || Nq == 0) return ATTN_OK;
  if (o == nullptr || lse == nullptr || q == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(lse) || !aligned16(q)) return ATTN_ERR_MISALIGNED;
  const long long rows = (long long)B * Hq * Nq;
  if (Nk == 0) return launch_fill_empty(o, lse, (size_t)rows, d, stream) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
  if (k == nullptr || v == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return ATTN_ERR_MISALIGNED;
  if ((long long)B * Hq > (1LL << 31) - 1) return ATTN_ERR_UNSUPPORTED;

  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)d);
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  // GQA with an even group: a CTA's two query tiles are two heads of one KV group at the
  // same rows (same keys, same mask, each K/V tile used by both); otherwise two adjacent
  // 128-row tiles of one head
  p.head_pairs = (p.G % 2 == 0) ? 1 : 0;
  p.num_pairs = p.head_pairs ? (Nq + 127) / 128 : (Nq + 255) / 256;
  p.num_sms = sm_count(current_device());
  // Packed documents: a unit's cost follows the document layout, so the units are dealt by
  // cost (sorted in every CTA) when they are few enough to sort in shared memory.
  p.sched = 0;
  if (mask_kind == ATTN_MASK_DOCUMENT_CAUSAL) {
    const long long U = (long long)p.num_pairs * B * (p.head_pairs ? Hq / 2 : Hq);
    const long long G = std::min<long long>(U, p.num_sms);
    if (U <= kSchedUnits && (U + G - 1) / G + 1 <= kSchedMax) p.sched = 1;
  }
  p.kscale = scale * kLog2e;
  p.softcap = softcap > 0.f ? softcap : 0.f;
  p.cap_scale = softcap > 0.f ? scale / softcap : 0.f;
  p.cap_log2 = softcap > 0.f ? softcap * kLog2e : 0.f;
  soft_cap_poly(p.cap_scale, p.cap_log2, p.cap_poly, p.cap_fast_max);
  p.mask = mask_params(mask_kind, window, doc_offsets, num_docs, Nq, Nk);
  p.alibi = alibi_slopes;
  p.kv_reverse = alibi_slopes != nullptr ? 1 : 0;
  if ((long long)p.num_pairs * B * Hq > (1LL << 31) - 1) return ATTN_ERR_UNSUPPORTED;
  p.err = error_word_ptr(current_device());
  if (p.err == nullptr) return ATTN_ERR_CUDA;

  CUtensorMap tq, tk, tv;
  if (!make_map_3d(&tq, q, d, Nq, (long long)B * Hq, 128) ||
      !make_map_3d(&tk, k, d, Nk, (long long)B * Hkv, 128) ||
      !make_map_3d(&tv, v, d, Nk, (long long)B * Hkv, 128))
    return ATTN_ERR_CUDA;
  return launch_attn_fwd(tq, tk, tv, p, d, stream) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" int attn_blockmap(int B, int Nq, int Nk, int mask_kind, int window,
                             const int* doc_offsets, int num_docs, unsigned char* map,
                             cudaStream_t stream) {
  if (B < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  int st = check_mask(mask_kind, window, doc_offsets, num_docs, Nq, Nk);
  if (st != ATTN_OK) return st;
  if (B == 0 || Nq == 0 || Nk == 0) return ATTN_OK;
  if (map == nullptr) return ATTN_ERR_INVALID_ARG;
  MaskParams m = mask_params(mask_kind, window, doc_offsets, num_docs, Nq, Nk);
  return launch_blockmap(m, B, Nq, Nk, map, stream) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" size_t attn_decode_workspace_bytes(int B, int Hq, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || d <= 0 || num_splits <= 0) return 0;
  const size_t rows = (size_t)B * Hq * num_splits;
  const size_t o_bytes = (rows * d * 4 + 255) & ~(size_t)255;
  return o_bytes + rows * 4;
}

extern "C" int attn_decode_default_splits(int B, int Hkv, int T, int device) {
  // Work items are (batch, kv head, split); a persistent grid of (SMs x resident CTAs)
  // slots walks them.  Take the smallest split count whose items fill the slots in whole
  // waves to within 1 %, keeping at least 128 keys per split.
  if (B <= 0 || Hkv <= 0 || T <= 0) return 1;
  const long long slots = (long long)sm_count(device) * 2;   // 2 resident CTAs at d=128, G<=8
  const long long heads = (long long)B * Hkv;
  const int max_splits = (int)std::max(1LL, std::min<long long>(256, (long long)T / 128));
  int best = 1;
  double best_eff = -1.0;
  for (int s = 1; s <= max_splits; ++s) {
    const long long items = heads * s;
    const long long waves = (items + slots - 1) / slots;
    const double eff = (double)items / (double)(waves * slots);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
    if (eff >= 0.99) break;
  }
  return best;
}

extern "C" int attn_decode_merge(const float* o_part, const float* lse_part, void* o, float* lse,
                                 long long rows, int num_splits, int d, cudaStream_t stream) {
  if (rows < 0 || num_splits < 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (rows == 0) return ATTN_OK;
  if (!o_part || !lse_part || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o_part) || !aligned16(o) || ((uintptr_t)lse_part & 3u) || ((uintptr_t)lse & 3u))
    return ATTN_ERR_MISALIGNED;
  return launch_merge(o_part, lse_part, o, lse, rows, num_splits, d, stream) == 0 ? ATTN_OK
                                                                                  : ATTN_ERR_CUDA;
}

extern "C" int attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                                   void* o, float* lse, int B, int Hq, int Hkv, int T, int d,
                                   float scale, int num_splits, void* workspace,
                                   size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || T < 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Hkv == 0 && Hq > 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv > 0 && Hq % Hkv != 0) return ATTN_ERR_UNSUPPORTED;
  if (std::isnan(scale)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0) return ATTN_OK;
  const int G = Hq / Hkv;
  if (G > 16) return ATTN_ERR_UNSUPPORTED;
  if (!q || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse)) return ATTN_ERR_MISALIGNED;
  if (T == 0) return launch_fill_empty(o, lse, (size_t)B * Hq, d, stream) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
  if (!k_cache || !v_cache) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return ATTN_ERR_MISALIGNED;
  const int dev = current_device();
  if (num_splits <= 0) num_splits = attn_decode_default_splits(B, Hkv, T, dev);
  if (num_splits > T) num_splits = T;
  const size_t need = attn_decode_workspace_bytes(B, Hq, d, num_splits);
  if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_MISALIGNED;
  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)d);

  DecParams p{};
  p.q = q;
  p.o_part = reinterpret_cast<float*>(workspace);
  const size_t rows = (size_t)B * Hq * num_splits;
  p.lse_part = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                        ((rows * d * 4 + 255) & ~(size_t)255));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.T = T;
  p.S = num_splits;
  p.num_items = B * Hkv * num_splits;
  p.kscale = scale * kLog2e;
  if ((long long)B * Hkv * num_splits > (1LL << 31) - 1) return ATTN_ERR_UNSUPPORTED;
  p.err = error_word_ptr(dev);
  if (p.err == nullptr) return ATTN_ERR_CUDA;

  CUtensorMap tk, tv;
  if (!make_map_3d(&tk, k_cache, d, T, (long long)B * Hkv, 64) ||
      !make_map_3d(&tv, v_cache, d, T, (long long)B * Hkv, 64))
    return ATTN_ERR_CUDA;
  const int slots = sm_count(dev) * decode_ctas_per_sm(d, G);
  const int grid = (int)std::min<long long>(p.num_items, slots);
  if (launch_decode_split(tk, tv, p, d, G, grid, stream) != 0) return ATTN_ERR_CUDA;
  return launch_merge(p.o_part, p.lse_part, o, lse, (long long)B * Hq, num_splits, d, stream) == 0
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

static int g_last_site = 0;

extern "C" int attn_get_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
  uint32_t word[2] = {0u, 0u};
  const uint32_t zero[2] = {0u, 0u};
  if (cudaMemcpyFromSymbol(word, g_error, sizeof(word)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (word[0] == 0) return ATTN_OK;
  if (cudaMemcpyToSymbol(g_error, zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  g_last_site = (int)word[1];
  return (word[0] & kErrWaitTimeout) ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_ERR_CUDA;
}

extern "C" int attn_last_error_site(void) { return g_last_site; }

extern "C" int attn_set_wait_limit_ns(unsigned long long ns) {
  const uint64_t v = ns;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  return cudaMemcpyToSymbol(g_error, &v, sizeof(v), 2 * sizeof(uint32_t)) == cudaSuccess
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

extern "C" int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                 const int* block_table, const int* seq_lens, void* o, float* lse,
                                 int B, int Hq, int Hkv, int num_pages, int page_size,
                                 int max_pages_per_seq, int d, float scale, int num_splits,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || num_pages < 0 || page_size <= 0 || max_pages_per_seq < 0)
    return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (page_size % 64 != 0) return ATTN_ERR_UNSUPPORTED;
  if (Hkv == 0 && Hq > 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv > 0 && Hq % Hkv != 0) return ATTN_ERR_UNSUPPORTED;
  if (std::isnan(scale)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0) return ATTN_OK;
  const int G = Hq / Hkv;
  if (G > 16) return ATTN_ERR_UNSUPPORTED;
  if (!q || !o || !lse || !seq_lens || !block_table) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse)) return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(seq_lens) & 3u) || (reinterpret_cast<uintptr_t>(block_table) & 3u))
    return ATTN_ERR_MISALIGNED;
  const long long t_cap = (long long)max_pages_per_seq * page_size;
  if (num_pages == 0 || t_cap == 0)
    return launch_fill_empty(o, lse, (size_t)B * Hq, d, stream) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
  if (!k_pages || !v_pages) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(k_pages) || !aligned16(v_pages)) return ATTN_ERR_MISALIGNED;
  if (t_cap > (1LL << 31) - 1 || (long long)num_pages * Hkv > (1LL << 31) - 1)
    return ATTN_ERR_UNSUPPORTED;
  const int dev = current_device();
  const int tiles = (int)((t_cap + 63) / 64);
  if (num_splits <= 0) num_splits = attn_decode_default_splits(B, Hkv, (int)t_cap, dev);
  if (num_splits > tiles) num_splits = tiles;
  const size_t need = attn_decode_workspace_bytes(B, Hq, d, num_splits);
  if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_MISALIGNED;
  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)d);

  DecParams p{};
  p.q = q;
  p.o_part = reinterpret_cast<float*>(workspace);
  const size_t rows = (size_t)B * Hq * num_splits;
  p.lse_part = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                        ((rows * d * 4 + 255) & ~(size_t)255));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.T = (int)t_cap;
  p.S = num_splits;
  if ((long long)B * Hkv * num_splits > (1LL << 31) - 1) return ATTN_ERR_UNSUPPORTED;
  p.num_items = B * Hkv * num_splits;
  p.kscale = scale * kLog2e;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.page_size = page_size;
  p.max_pages = max_pages_per_seq;
  p.err = error_word_ptr(dev);
  if (p.err == nullptr) return ATTN_ERR_CUDA;

  CUtensorMap tk, tv;
  if (!make_map_3d(&tk, k_pages, d, page_size, (long long)num_pages * Hkv, 64) ||
      !make_map_3d(&tv, v_pages, d, page_size, (long long)num_pages * Hkv, 64))
    return ATTN_ERR_CUDA;
  const int slots = sm_count(dev) * decode_ctas_per_sm(d, G);
  const int grid = (int)std::min<long long>(p.num_items, slots);
  if (launch_decode_split(tk, tv, p, d, G, grid, stream) != 0) return ATTN_ERR_CUDA;
  return launch_merge(p.o_part, p.lse_part, o, lse, (long long)B * Hq, num_splits, d, stream) == 0
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

extern "C" size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq) {
  if (B <= 0 || Hq <= 0 || Nq <= 0) return 0;
  const size_t rows = (size_t)B * Hq * Nq;
  return 2 * ((rows * 4 + 255) & ~(size_t)255);
}

extern "C" int attn_bwd(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                        int Hq, int Hkv, int Nq, int Nk, int d, float scale, int mask_kind,
                        int window, float softcap, const int* doc_offsets, int num_docs,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return attn_bwd_alibi(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale,
                        mask_kind, window, softcap, doc_offsets, num_docs, nullptr, workspace,
                        workspace_bytes, stream);
}

extern "C" int attn_bwd_alibi(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                              int mask_kind, int window, float softcap, const int* doc_offsets,
                              int num_docs, const float* alibi_slopes, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(alibi_slopes) & 3u) return ATTN_ERR_MISALIGNED;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Hkv == 0 && Hq > 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv > 0 && Hq % Hkv != 0) return ATTN_ERR_UNSUPPORTED;
  int st = check_mask(mask_kind, window, doc_offsets, num_docs, Nq, Nk);
  if (st != ATTN_OK) return st;
  if (std::isnan(scale) || std::isnan(softcap)) return ATTN_ERR_INVALID_ARG;
  if (softcap > 0.f && alibi_slopes != nullptr) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || Hq == 0 || (Nq == 0 && Nk == 0)) return ATTN_OK;
  const void* ptrs[] = {q, k, v, o, dout, lse, dq, dk, dv};
  const int needed[] = {Nq > 0, Nk > 0, Nk > 0, Nq > 0, Nq > 0, Nq > 0, Nq > 0, Nk > 0, Nk > 0};
  for (int i = 0; i < 9; ++i) {
    if (!needed[i]) continue;
    if (ptrs[i] == nullptr) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(ptrs[i])) return ATTN_ERR_MISALIGNED;
  }
  const size_t rows = (size_t)B * Hq * Nq;
  const size_t need = attn_bwd_workspace_bytes(B, Hq, Nq);
  if (Nq > 0 && (workspace == nullptr || workspace_bytes < need)) return ATTN_ERR_WORKSPACE;
  if (Nq > 0 && !aligned16(workspace)) return ATTN_ERR_MISALIGNED;
  if ((long long)B * Hq > (1LL << 31) - 1 || (long long)B * Hkv * ((Nk + 127) / 128) > (1LL << 31) - 1 ||
      (long long)B * Hq * ((Nq + 127) / 128) > (1LL << 31) - 1)
    return ATTN_ERR_UNSUPPORTED;
  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)d);
  const int dev = current_device();

  BwdParams p{};
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dvec = reinterpret_cast<float*>(workspace);
  p.l2 = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + need / 2);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  p.kscale = scale * kLog2e;
  p.scale = scale;
  p.mask = mask_params(mask_kind, window, doc_offsets, num_docs, Nq, Nk);
  p.alibi = alibi_slopes;
  p.cap_scale = softcap > 0.f ? scale / softcap : 0.f;
  p.cap_log2 = softcap > 0.f ? softcap * kLog2e : 0.f;
  soft_cap_poly(p.cap_scale, p.cap_log2, p.cap_poly, p.cap_fast_max);
  p.err = error_word_ptr(dev);
  if (p.err == nullptr) return ATTN_ERR_CUDA;
  if (Nq > 0 && launch_bwd_rowdot(o, dout, lse, const_cast<float*>(p.dvec),
                                  const_cast<float*>(p.l2), (long long)rows, d, stream) != 0)
    return ATTN_ERR_CUDA;

  // With no query rows dK = dV = 0; with no keys dQ = 0 (the kernels write these too, but
  // their maps need a non-empty tensor).
  CUtensorMap tq, tdo, tk, tv;
  if (Nq == 0 || Nk == 0) {
    if (Nk > 0) {
      if (cudaMemsetAsync(dk, 0, (size_t)B * Hkv * Nk * d * 2, stream) != cudaSuccess ||
          cudaMemsetAsync(dv, 0, (size_t)B * Hkv * Nk * d * 2, stream) != cudaSuccess)
        return ATTN_ERR_CUDA;
    }
    if (Nq > 0 && cudaMemsetAsync(dq, 0, rows * d * 2, stream) != cudaSuccess)
      return ATTN_ERR_CUDA;
    return ATTN_OK;
  }
  if (!make_map_3d(&tq, q, d, Nq, (long long)B * Hq, 128) ||
      !make_map_3d(&tdo, dout, d, Nq, (long long)B * Hq, 128) ||
      !make_map_3d(&tk, k, d, Nk, (long long)B * Hkv, 128) ||
      !make_map_3d(&tv, v, d, Nk, (long long)B * Hkv, 128))
    return ATTN_ERR_CUDA;
  return launch_attn_bwd(tq, tdo, tk, tv, p, d, stream) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" int attn_quantize_fp8(const void* x, void* out, float* scales, int B, int H, int N,
                                 int d, int block_rows, int transpose, int n_pad,
                                 const float* signs, cudaStream_t stream) {
  if (B < 0 || H < 0 || N < 0 || block_rows <= 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (transpose && n_pad < N) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return ATTN_OK;
  if (!x || !out || !scales) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(scales) & 3u) ||
      (reinterpret_cast<uintptr_t>(signs) & 3u))
    return ATTN_ERR_MISALIGNED;
  if (!transpose && (reinterpret_cast<uintptr_t>(out) & 3u)) return ATTN_ERR_MISALIGNED;
  uint32_t* err = error_word_ptr(current_device());
  if (err == nullptr) return ATTN_ERR_CUDA;
  // row-major blocks of at most 128 rows take tiled copies (the other layouts plain loads)
  CUtensorMap tx;
  const bool tiled = !transpose && block_rows <= 128 &&
                     make_map_3d(&tx, x, d, N, (long long)B * H, block_rows);
  return launch_quantize_e4m3(tiled ? &tx : nullptr, x, out, scales, B, H, N, d, block_rows,
                              transpose, n_pad, signs, err, sm_count(current_device()),
                              stream) == 0
             ? ATTN_OK
             : ATTN_ERR_CUDA;
}

extern "C" int attn_fwd_fp8(const void* q8, const void* k8, const void* vt8,
                            const float* q_scales, const float* k_scales, const float* v_scales,
                            void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk,
                            int nk_pad, int d, float scale, int mask_kind, int window,
                            const int* doc_offsets, int num_docs, cudaStream_t stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Hkv == 0 && Hq > 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv > 0 && Hq % Hkv != 0) return ATTN_ERR_UNSUPPORTED;
  int st = check_mask(mask_kind, window, doc_offsets, num_docs, Nq, Nk);
  if (st != ATTN_OK) return st;
  if (std::isnan(scale)) return ATTN_ERR_INVALID_ARG;
  if (nk_pad < Nk || (nk_pad & 15)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0 || Nq == 0) return ATTN_OK;
  if (!o || !lse || !q8 || !q_scales) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(lse) || !aligned16(q8)) return ATTN_ERR_MISALIGNED;
  const long long rows = (long long)B * Hq * Nq;
  if (Nk == 0) return launch_fill_empty(o, lse, (size_t)rows, d, stream) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
  if (!k8 || !vt8 || !k_scales || !v_scales) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(k8) || !aligned16(vt8)) return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(q_scales) | reinterpret_cast<uintptr_t>(k_scales) |
       reinterpret_cast<uintptr_t>(v_scales)) & 3u)
    return ATTN_ERR_MISALIGNED;
  if ((long long)B * Hq > (1LL << 31) - 1) return ATTN_ERR_UNSUPPORTED;

  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)d);
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  // GQA with an even group: a CTA's two query tiles are two heads of one KV group at the
  // same rows (same keys, same mask, each K/V tile used by both); otherwise two adjacent
  // 128-row tiles of one head
  p.head_pairs = (p.G % 2 == 0) ? 1 : 0;
  p.num_pairs = p.head_pairs ? (Nq + 127) / 128 : (Nq + 255) / 256;
  p.num_sms = sm_count(current_device());
  p.kscale = scale * kLog2e;
  p.mask = mask_params(mask_kind, window, doc_offsets, num_docs, Nq, Nk);
  p.q_scales = q_scales;
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  p.nqt = (Nq + 127) / 128;
  p.nkt = (Nk + 127) / 128;
  if ((long long)p.num_pairs * B * Hq > (1LL << 31) - 1) return ATTN_ERR_UNSUPPORTED;
  p.err = error_word_ptr(current_device());
  if (p.err == nullptr) return ATTN_ERR_CUDA;

  CUtensorMap tq, tk, tv;
  if (!make_map_3d_u8(&tq, q8, d, d, Nq, (long long)B * Hq, 128) ||
      !make_map_3d_u8(&tk, k8, d, d, Nk, (long long)B * Hkv, 128) ||
      !make_map_3d_u8(&tv, vt8, Nk, nk_pad, d, (long long)B * Hkv, d))
    return ATTN_ERR_CUDA;
  return launch_attn_fwd(tq, tk, tv, p, d, stream) == 0 ? ATTN_OK : ATTN_ERR_CUDA;
}
