// Split-KV decode for callers that cannot allocate device memory.
//
// attn_decode_splitkv needs a caller-provided fp32 workspace for the per-split partial
// results.  Some callers have no way to provide one: a plugin or extension that runs inside
// a host application which owns every device allocation, code that must not allocate while a
// stream is being captured into a CUDA graph, or a real-time loop whose memory budget is fixed
// up front and forbids cudaMalloc/cudaFree on the hot path.  For them this file keeps a
// workspace inside the library's own device image -- a file-scope __device__ array loaded
// with the module -- and runs the unchanged split-KV path on it.  The caller still passes
// q, the caches and the outputs.
//
// Limits and rules of use:
//   * the array is kNoAllocWorkspaceBytes (32 MiB); a valid request whose partials would not
//     fit (B * Hq * splits * (d + 1) * 4 bytes, plus alignment) is rejected with
//     ATTN_ERR_WORKSPACE before anything runs (invalid arguments get attn_decode_splitkv's
//     own statuses first);
//   * every GPU that loads the library holds the array until the process exits;
//   * all calls share the one array per device, so two calls that overlap on the GPU (other
//     streams, other threads) race on it; serialise them on one stream;
//   * the array keeps the last call's partials; nothing in it has to start at zero because
//     every partial the merge reads is written earlier in the same call;
//   * in host code the array's name is only a host-side stand-in, so its device address is
//     looked up once per device with cudaGetSymbolAddress, with that device current; the
//     first call on each device performs this lookup and should therefore happen before any
//     stream capture.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"

namespace {

constexpr size_t kNoAllocWorkspaceBytes = 32ull << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_workspace[kNoAllocWorkspaceBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the workspace on `device` (which must be current); nullptr on failure.
void* noalloc_workspace(int device) {
  if (device < 0 || device >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[device] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_workspace) != cudaSuccess) return nullptr;
    g_noalloc_addr[device] = ptr;
  }
  return g_noalloc_addr[device];
}

}  // namespace

extern "C" int attn_decode_splitkv_noalloc(const void* q, const void* k_cache,
                                           const void* v_cache, void* o, float* lse, int B,
                                           int Hq, int Hkv, int T, int d, float scale,
                                           int num_splits, cudaStream_t stream) {
  // The argument checks of attn_decode_splitkv come first, in its order, so that an invalid
  // request gets the same status from both entry points whatever its size.
  if (B < 0 || Hq < 0 || Hkv < 0 || T < 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Hkv == 0 && Hq > 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv > 0 && Hq % Hkv != 0) return ATTN_ERR_UNSUPPORTED;
  if (std::isnan(scale)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0 || T == 0) {
    // nothing needs partials: the regular entry point handles these without a workspace
    return attn_decode_splitkv(q, k_cache, v_cache, o, lse, B, Hq, Hkv, T, d, scale,
                               num_splits, nullptr, 0, stream);
  }
  if (Hq / Hkv > 16) return ATTN_ERR_UNSUPPORTED;
  if (!q || !o || !lse || !k_cache || !v_cache) return ATTN_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
  if (misaligned(q) || misaligned(o) || misaligned(lse) || misaligned(k_cache) ||
      misaligned(v_cache))
    return ATTN_ERR_MISALIGNED;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return ATTN_ERR_CUDA;
  int splits = num_splits;
  if (splits <= 0) splits = attn_decode_default_splits(B, Hkv, T, device);
  if (splits > T) splits = T;
  const size_t need = attn_decode_workspace_bytes(B, Hq, d, splits);
  if (need == 0 || need > kNoAllocWorkspaceBytes) return ATTN_ERR_WORKSPACE;
  void* ws = noalloc_workspace(device);
  if (ws == nullptr) return ATTN_ERR_CUDA;
  return attn_decode_splitkv(q, k_cache, v_cache, o, lse, B, Hq, Hkv, T, d, scale, splits, ws,
                             kNoAllocWorkspaceBytes, stream);
}
