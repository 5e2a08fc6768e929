/*
 * io_aware_softmax_b200 -- exact fused attention on NVIDIA B200 (sm_100a), C ABI.
 *
 * What is computed (the plain definition the kernels reproduce up to rounding):
 *   O = softmax(scale * Q K^T + mask) V, and the row log-sum-exp LSE = ln sum_j exp(s_ij)
 * ("PyTorch FlexAttention 도입 분석", section 1; "FlashAttention 논문 분석: IO-Aware Exact
 * Attention", section "수학적 정의"; the row statistics m and l that the forward keeps for a
 * recomputing backward, section "Recomputation 전략").  The score matrix S and the
 * probabilities P never reach device memory: the softmax is taken tile by tile with the
 * online rescaling of "Online Softmax와 블록 단위 누적" / "알고리즘 의사코드" on the same page.
 *
 * Conventions shared by every entry point:
 *   - Tensors are caller-owned DEVICE memory, contiguous, row-major in the order given
 *     ([B, H, N, d] as in PyTorch, "사례 2: 텐서 형태 불일치" on the FlashAttention page).
 *     bf16 arrays are passed as void*.  Every pointer must be 16-byte aligned.
 *     Each array must hold at least the elements its stated shape implies: the library
 *     sees only pointers and sizes, so it cannot check an allocation's extent (the Python
 *     binding checks every tensor's shape, dtype and device before it calls in).
 *   - The compute entry points (attn_fwd, attn_fwd_alibi, attn_bwd, attn_bwd_alibi,
 *     attn_quantize_fp8, attn_fwd_fp8, attn_blockmap, attn_decode_splitkv, attn_decode_paged,
 *     attn_decode_merge) are asynchronous on `stream`; they never synchronise, never allocate
 *     and keep no state across calls except a per-process cache of device attributes, so
 *     they may be recorded into a CUDA graph with fixed shapes ("CUDA 그래프와의 호환성").
 *     attn_get_device_status and attn_set_wait_limit_ns synchronise.
 *   - Arguments are validated before anything is launched; an unsupported case returns
 *     ATTN_ERR_UNSUPPORTED and nothing runs -- there is no fallback path ("3.7 어텐션 II",
 *     section 3.7.3, on diagnosing silent fallbacks: here the failure is the diagnosis).
 *   - Kernels never hang: every wait inside them is bounded.  A wait that runs out records
 *     a device-side error and the kernel returns; attn_get_device_status() reports it.
 */
#ifndef IO_AWARE_SOFTMAX_B200_ATTN_H
#define IO_AWARE_SOFTMAX_B200_ATTN_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Mask hooks ("PyTorch FlexAttention 도입 분석", section 2: score_mod / mask applied to each
 * scalar score right after Q.K^T).  Every kind other than NONE needs Nq == Nk. */
typedef enum {
  ATTN_MASK_NONE = 0,             /* every key visible                                    */
  ATTN_MASK_CAUSAL = 1,           /* kv <= q                                               */
  ATTN_MASK_SLIDING_CAUSAL = 2,   /* 0 <= q - kv <= window (window + 1 keys incl. self)    */
  ATTN_MASK_DOCUMENT_CAUSAL = 3,  /* same packed document AND kv <= q                      */
  ATTN_MASK_SLIDING = 4           /* |q - kv| <= window, no causality (2 window + 1 keys)  */
} attn_mask_kind;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1,      /* null pointer, negative size, bad mask parameters       */
  ATTN_ERR_UNSUPPORTED = -2,      /* valid request this library does not implement          */
  ATTN_ERR_MISALIGNED = -3,       /* a pointer is not 16-byte aligned                       */
  ATTN_ERR_CUDA = -4,             /* a CUDA runtime/driver call failed                      */
  ATTN_ERR_DEVICE_TIMEOUT = -5,   /* a kernel's bounded wait ran out (see get_device_status)*/
  ATTN_ERR_WORKSPACE = -6         /* workspace missing or too small                         */
} attn_status;

typedef enum { ATTN_TILE_EMPTY = 0, ATTN_TILE_PARTIAL = 1, ATTN_TILE_FULL = 2 } attn_tile_class;

/*
 * attn_fwd -- fused prefill attention forward.
 * Defining passages: FlashAttention page, "알고리즘 의사코드" (tiled forward returning O, m, l);
 * "3.7 어텐션 II", 3.7.5 (GQA/MQA: query-head groups share a KV head; sliding window;
 * soft-cap as a kernel flag) and 3.7.6 (packed documents by cumulative boundaries).
 *
 *   q        bf16 [B, Hq,  Nq, d]     k, v  bf16 [B, Hkv, Nk, d]
 *   o        bf16 [B, Hq,  Nq, d]     (written)   lse  fp32 [B, Hq, Nq] natural log (written)
 *   d        64 or 128; Hq % Hkv == 0; query head h reads KV head h / (Hq / Hkv)
 *   scale    multiplies q.k; <= 0 selects 1/sqrt(d)
 *   mask_kind, window   see attn_mask_kind; window >= 0 for SLIDING_CAUSAL and SLIDING
 *   softcap  > 0: score s (already scaled) becomes softcap * tanh(s / softcap); <= 0: off
 *   doc_offsets, num_docs   DOCUMENT_CAUSAL only: device int32 [num_docs + 1], with
 *            doc_offsets[0] = 0, non-decreasing, doc_offsets[num_docs] = Nk; the same
 *            documents apply to every batch entry.  Ignored for other masks.
 * A row with no visible key gets O = 0 and LSE = -inf.  Outputs are rounded to bf16 (RNE).
 * Errors: INVALID_ARG, UNSUPPORTED (d not in {64,128}; Hq % Hkv != 0; a mask with
 * Nq != Nk), MISALIGNED, CUDA.  Empty problems (B, Hq or Nq == 0) return ATTN_OK at once.
 */
ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, float scale, int mask_kind, int window,
             float softcap, const int* doc_offsets, int num_docs, cudaStream_t stream);

/*
 * attn_fwd_alibi -- attn_fwd with the ALiBi positional bias fused into the score
 * ("3.7 어텐션 II", 3.7.5: a distance-based bias added before the softmax, fused instead of
 * passed as a mask tensor).  Query head h adds -alibi_slopes[h] * |q - kv| (natural-log
 * units) to the score after scaling and soft-capping and before the mask.
 *   alibi_slopes  device fp32 [Hq], 4-byte aligned, read by the kernel; NULL behaves as
 *                 attn_fwd.  Every other argument, the outputs and the errors as attn_fwd,
 *                 plus UNSUPPORTED for a bias together with softcap > 0.
 */
ATTN_API int attn_fwd_alibi(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int mask_kind,
             int window, float softcap, const int* doc_offsets, int num_docs,
             const float* alibi_slopes, cudaStream_t stream);

/*
 * attn_bwd -- backward pass of attn_fwd: dQ, dK, dV from (q, k, v, o, dout, lse).
 * Defining passages: FlashAttention page, "Recomputation 전략" (S and P are recomputed block
 * by block from the saved row statistics instead of keeping an N x N matrix) -- here from
 * the natural-log LSE attn_fwd returns; the gradients are those of the definition:
 * dV = P^T dO, dP = dO V^T, dS = P (dP - rowsum(dO * O)), dQ = scale dS K,
 * dK = scale dS^T Q, a KV head's dK and dV summing over its query-head group.
 *
 *   q, k, v, o, lse   as attn_fwd (o and lse: attn_fwd's outputs for these inputs)
 *   dout         bf16 [B, Hq, Nq, d]   gradient of the loss with respect to o
 *   dq           bf16 [B, Hq, Nq, d]   dk, dv  bf16 [B, Hkv, Nk, d]   (written)
 *   mask_kind, window, doc_offsets, num_docs, scale, softcap   as attn_fwd (with a soft-cap
 *                the capped score y = c tanh(x / c) passes dy (1 - tanh^2(x / c)) on to x)
 *   workspace    device, 16-byte aligned, attn_bwd_workspace_bytes(B, Hq, Nq) bytes (the
 *                per-row rowsum(dO * O) and base-2 LSE); contents are scratch
 * Three kernel launches on `stream`, no host synchronisation.  Rows with no visible key
 * (LSE = -inf) contribute nothing; keys no query sees get dK = dV = 0.
 * Errors: as attn_fwd, plus WORKSPACE.
 */
ATTN_API size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq);
ATTN_API int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
             int Nk, int d, float scale, int mask_kind, int window, float softcap,
             const int* doc_offsets, int num_docs, void* workspace, size_t workspace_bytes,
             cudaStream_t stream);

/*
 * attn_bwd_alibi -- attn_bwd for scores that carry the ALiBi bias of attn_fwd_alibi
 * ("3.7 어텐션 II", 3.7.5).  The bias depends on positions only, so the gradients keep the
 * form of attn_bwd with P recomputed from the biased scores:
 * P_ij = exp(scale q_i.k_j - slope_h |i - j| - LSE_i).
 *   alibi_slopes  device fp32 [Hq], 4-byte aligned (the slopes given to attn_fwd_alibi;
 *                 o and lse must come from that call); NULL behaves as attn_bwd.
 * Every other argument, the workspace and the errors as attn_bwd, plus UNSUPPORTED for
 * slopes together with softcap > 0 (as attn_fwd_alibi).
 */
ATTN_API int attn_bwd_alibi(const void* q, const void* k, const void* v, const void* o,
             const void* dout, const float* lse, void* dq, void* dk, void* dv, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, float scale, int mask_kind, int window,
             float softcap, const int* doc_offsets, int num_docs, const float* alibi_slopes,
             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * attn_quantize_fp8 -- block quantization to E4M3 ("FlashAttention 논문 분석", section
 * "FP8 지원과 정확도 유지": an independent scale per block; Q and K optionally multiplied by a
 * random orthogonal matrix first, which leaves Q K^T unchanged).
 *   x        bf16 [B, H, N, d], d in {64, 128}
 *   signs    NULL, or device fp32 [d] of +-1: rows become (x * signs) H / sqrt(d), H the
 *            Sylvester Hadamard matrix (use the same signs for Q and K)
 *   block_rows  rows per scale; scales fp32 [B, H, ceil(N / block_rows)] (written):
 *            amax / 448 of the (rotated) block, 1 for an all-zero block
 *   out      E4M3 codes (written) of x * (448 / amax), round to nearest even, saturating:
 *            transpose = 0: [B, H, N, d]; transpose = 1: [B, H, d, n_pad] with columns
 *            [N, n_pad) zero (the layout attn_fwd_fp8 takes for V)
 * Errors: INVALID_ARG, UNSUPPORTED (d), MISALIGNED (x 16 bytes; scales, signs and a
 * row-major out 4 bytes), CUDA.
 */
ATTN_API int attn_quantize_fp8(const void* x, void* out, float* scales, int B, int H, int N, int d,
                      int block_rows, int transpose, int n_pad, const float* signs,
                      cudaStream_t stream);

/*
 * attn_fwd_fp8 -- attn_fwd on E4M3 inputs (the FP8 tensor-core path of "FlashAttention 논문
 * 분석", sections "FP8 텐서 코어" and "FP8 지원과 정확도 유지").  The result is attention of
 * the dequantized values: Q = q8 * q_scales (per 128-row block), K = k8 * k_scales (per
 * 128-row block), V = vt8^T * v_scales (per head).  Both products run on E4M3 operands;
 * P is rounded to E4M3 (as 64 P, the lazy-rescale bound being 2^2).
 *   q8       E4M3 [B, Hq, Nq, 128]            q_scales  fp32 [B, Hq, ceil(Nq / 128)]
 *   k8       E4M3 [B, Hkv, Nk, 128]           k_scales  fp32 [B, Hkv, ceil(Nk / 128)]
 *   vt8      E4M3 [B, Hkv, 128, nk_pad] (V transposed; nk_pad >= Nk, a multiple of 16)
 *   v_scales fp32 [B, Hkv]
 *   o, lse, scale, masks as attn_fwd (no soft-cap); d must be 128.
 * Errors: as attn_fwd; UNSUPPORTED for d != 128.
 */
ATTN_API int attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* q_scales,
                 const float* k_scales, const float* v_scales, void* o, float* lse, int B,
                 int Hq, int Hkv, int Nq, int Nk, int nk_pad, int d, float scale, int mask_kind,
                 int window, const int* doc_offsets, int num_docs, cudaStream_t stream);

/*
 * attn_blockmap -- 128x128 block-sparsity map of a mask ("PyTorch FlexAttention 도입 분석",
 * section 2: BlockMask precomputed in 128 x 128 chunks so empty tiles are skipped).
 *   map  device uint8 [B, ceil(Nq/128), ceil(Nk/128)] (written): ATTN_TILE_EMPTY when no
 *        (q, kv) pair of the tile is visible, ATTN_TILE_FULL when all are, else PARTIAL.
 *        Only pairs with q < Nq and kv < Nk count.
 * Mask arguments and errors as attn_fwd.
 */
ATTN_API int attn_blockmap(int B, int Nq, int Nk, int mask_kind, int window, const int* doc_offsets,
                  int num_docs, unsigned char* map, cudaStream_t stream);

/*
 * Split-KV decode ("3.7 어텐션 II", 3.7.4: one query token against the whole KV cache; the
 * cache axis is split, every split produces partial (m, l, O), and the partials are merged
 * by the rescaling recurrence).
 *
 * attn_decode_workspace_bytes: bytes of device workspace attn_decode_splitkv needs for
 *   num_splits splits (fp32 partial O [B, Hq, S, d] and LSE [B, Hq, S]).
 * attn_decode_default_splits: the split count that fills every SM of `device` with whole
 *   waves of work items for B * Hkv KV heads and cache length T (>= 1).
 * attn_decode_splitkv:
 *   q        bf16 [B, Hq, 1, d]           k_cache, v_cache  bf16 [B, Hkv, T, d] contiguous
 *   o        bf16 [B, Hq, 1, d] (written) lse fp32 [B, Hq, 1] natural log (written)
 *   scale    <= 0 selects 1/sqrt(d); num_splits <= 0 selects attn_decode_default_splits
 *   workspace, workspace_bytes  caller-owned device scratch, >= attn_decode_workspace_bytes,
 *            16-byte aligned; its contents on return are the per-split partials.  Split s
 *            covers the 64-row tiles [s n / S, (s + 1) n / S) of the n = ceil(T / 64) tiles
 *            (rows past T excluded), so no tile is read by two splits.
 *   No mask (every cached key is visible).  Hq / Hkv <= 16, d in {64, 128}.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA.  T == 0 writes O = 0 and
 * LSE = -inf.
 */
ATTN_API size_t attn_decode_workspace_bytes(int B, int Hq, int d, int num_splits);
ATTN_API int attn_decode_default_splits(int B, int Hkv, int T, int device);
ATTN_API int attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, void* o,
                        float* lse, int B, int Hq, int Hkv, int T, int d, float scale,
                        int num_splits, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/*
 * attn_decode_splitkv_noalloc -- attn_decode_splitkv for callers that cannot allocate
 * device memory (a plugin inside a host that owns every allocation, code that must not
 * allocate while a stream is captured, a loop with a fixed memory budget).  This entry point
 * has no counterpart in the pages; it only moves the workspace into the library.
 *   Arguments as attn_decode_splitkv without workspace/workspace_bytes: the split partials
 *   live in a library-owned device array of 32 MiB that every GPU loading the library holds
 *   until exit.  Requests whose partials exceed it (B * Hq * splits * (d + 1) * 4 bytes plus
 *   alignment) return ATTN_ERR_WORKSPACE before anything runs.
 *   All calls on a device share that array and it keeps the last call's contents: calls that
 *   overlap on the GPU race, so issue them on one stream.  The first call on each device looks
 *   up the array's device address (with that device current); make that first call before
 *   any stream capture.  No allocation happens in any call.
 * Errors: as attn_decode_splitkv, checked in the same order first, so an invalid request gets
 * the same status from both; WORKSPACE then means a valid request too large for the array.
 */
ATTN_API int attn_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         void* o, float* lse, int B, int Hq, int Hkv, int T,
                                         int d, float scale, int num_splits,
                                         cudaStream_t stream);

/*
 * attn_decode_paged -- split-KV decode over paged, variable-length KV caches
 * ("3.7 어텐션 II", 3.7.4: decode attention goes with paged KV management and in-flight
 * batching; 3.7.8: PagedAttention keeps the cache in pages; 3.7.6: the sequences of a
 * batch keep their own lengths).  Sequence b attends to its first seq_lens[b] cache rows;
 * logical row t of sequence b is row (t % page_size) of physical page
 * block_table[b * max_pages_per_seq + t / page_size].
 *
 *   q             bf16 [B, Hq, 1, d]            o bf16 [B, Hq, 1, d], lse fp32 [B, Hq, 1]
 *   k_pages, v_pages  bf16 [num_pages, Hkv, page_size, d] (one page holds page_size rows
 *                 of every KV head); page_size a multiple of 64
 *   block_table   device int32 [B, max_pages_per_seq]; entries in [0, num_pages) for the
 *                 pages a sequence uses (entries past its length are not read)
 *   seq_lens      device int32 [B]; values are clamped to [0, max_pages_per_seq * page_size]
 *   num_splits, workspace, workspace_bytes  as attn_decode_splitkv; splits cut each
 *                 sequence at 64-row tile boundaries (<= 0: attn_decode_default_splits for
 *                 max_pages_per_seq * page_size rows)
 * A sequence of length 0 gets O = 0 and LSE = -inf.  A page index outside [0, num_pages)
 * reads zeros (the copy engine fills rows outside the cache) rather than faulting.
 * A contiguous cache with per-sequence lengths is the case num_pages = B,
 * page_size = T (rounded up to 64), block_table[b] = {b}.
 * Errors: INVALID_ARG, UNSUPPORTED (d not in {64,128}; Hq % Hkv != 0; Hq / Hkv > 16;
 * page_size % 64 != 0), MISALIGNED (16 bytes for bf16 arrays and workspace, 4 for the int
 * arrays), WORKSPACE, CUDA.
 */
ATTN_API int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                      const int* block_table, const int* seq_lens, void* o, float* lse, int B,
                      int Hq, int Hkv, int num_pages, int page_size, int max_pages_per_seq, int d,
                      float scale, int num_splits, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream);

/*
 * attn_decode_merge -- merge S partial results per row by the rescaling rule ("3.7 어텐션
 * II", 3.7.4): L = max_s LSE_s, w_s = exp(LSE_s - L), O = sum_s w_s O_s / sum_s w_s,
 * LSE = L + ln sum_s w_s.  Partials with LSE = -inf have weight 0.
 *   o_part fp32 [rows, S, d] (each partial normalised by its own sum); lse_part fp32
 *   [rows, S]; o bf16 [rows, d] (written); lse fp32 [rows] (written).  d in {64, 128}.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, CUDA.
 */
ATTN_API int attn_decode_merge(const float* o_part, const float* lse_part, void* o, float* lse,
                      long long rows, int num_splits, int d, cudaStream_t stream);

/*
 * attn_get_device_status -- synchronises `stream`, then returns and clears the device-side
 * error word of the current device: ATTN_OK, ATTN_ERR_DEVICE_TIMEOUT (a bounded wait in a
 * kernel ran out; attn_last_error_site() names which), or ATTN_ERR_CUDA if the
 * synchronisation itself failed.
 */
ATTN_API int attn_get_device_status(cudaStream_t stream);
ATTN_API int attn_last_error_site(void);

/*
 * attn_set_wait_limit_ns -- sets, on the current device, how long a kernel's pipeline waits
 * (a warp waiting for a tile, a product or a free buffer) may last before the kernel gives up
 * and reports ATTN_ERR_DEVICE_TIMEOUT; 0 restores the built-in 0.5 s.  The waits of a
 * kernel's teardown (for its own copies and products still in flight) keep the full limit,
 * so a kernel that gave up still exits cleanly and later calls run normally.  It exists to
 * exercise the failure path ("3.7 어텐션 II", 3.7.3: a failure is reported, never hidden): a
 * limit of a few nanoseconds makes the first wait that is not already satisfied run out.
 * It synchronises the device first; call it with no call of this library in flight.
 * Errors: CUDA.
 */
ATTN_API int attn_set_wait_limit_ns(unsigned long long ns);

/* Human-readable name of a status code (static storage). */
ATTN_API const char* attn_status_string(int status);

/* Library ABI version (major * 100 + minor). */
ATTN_API int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* IO_AWARE_SOFTMAX_B200_ATTN_H */
