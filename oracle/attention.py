"""Plain, slow, obviously correct fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it. It shares no code with the CUDA
library (no kernels, headers, helpers, tables or constants); the two meet only through
the seeded input generators in ``workloads/``.

What it computes, and where that is written down (pages cited by title and section):

* Scores, softmax, output -- the definition ``softmax(Q K^T / sqrt(d_k)) V``:
  "PyTorch FlexAttention 도입 분석", section 1 (the attention formula);
  "FlashAttention 논문 분석: IO-Aware Exact Attention", section "수학적 정의" and the
  ``standard_attention`` listing under "IO 병목의 실체" (scores, masked_fill with -inf,
  softmax over the last axis, matmul with V);
  "어텐션 최적화: FlashAttention과 희소 어텐션", section "핵심 수식" and Steps 1-3
  (S = QK^T/sqrt(d_k); rows of A sum to 1; output_i = sum_j A_ij V_j).
* Masked entries are -inf before the softmax and so get probability 0:
  "Attention 최적화가 어려운 이유", section "Attention의 계산 흐름" (causal mask);
  "어텐션 최적화: FlashAttention과 희소 어텐션", Step 4 (E_ij = -inf for j not in S_i).
* score_mod hooks applied to the scaled score right after QK^T: the FlexAttention page,
  section 2 (``sliding_window_mod``: keep the score where |q_idx - kv_idx| <= 1024, else
  -inf); tanh soft-capping and document-boundary masking are named as kernel features in
  the FlexAttention page's opening section and in "3.7 어텐션 II", section 3.7.5.
* Row statistics m and l returned with O for the backward pass, so the row log-sum-exp
  is m + ln(l): FlashAttention page, sections "Recomputation 전략" and
  "알고리즘 의사코드".
* GQA/MQA: a group of query heads shares one KV head, never a copy:
  "3.7 어텐션 II", section 3.7.5; FlashAttention page, "사례 4: GQA/MQA 지원 문제".
* Packed documents delimited by cumulative boundaries (``cu_seqlens``):
  "3.7 어텐션 II", section 3.7.6.
* ALiBi: a distance-based positional bias added to the score before the softmax, fused in
  the kernel rather than passed as a mask tensor: "3.7 어텐션 II", section 3.7.5
  ("ALiBi·위치 바이어스").  The symmetric (non-causal) window is the FlexAttention page's
  ``sliding_window_mod`` as written, |q_idx - kv_idx| <= window.
* The tiled online-softmax form (normalised-O update with alpha = exp(m_old - m_new),
  beta = exp(m_local - m_new)): FlashAttention page, sections "Online Softmax와 블록 단위
  누적" and "알고리즘 의사코드".
* Backward pass: S and P are recomputed from the saved row statistics rather than kept
  from the forward pass: FlashAttention page, "Recomputation 전략"; the gradient formulas
  are the calculus of the definition (``attention_backward``).
* Split-KV decoding: each split produces partial (m, l, O) and the splits are combined by
  the same rescaling recurrence: "3.7 어텐션 II", section 3.7.4 (FlashDecoding).
* Paged, variable-length KV caches for decode (in-flight batching with a page table,
  PagedAttention): "3.7 어텐션 II", sections 3.7.4 and 3.7.8; the sequences of a batch have
  their own lengths, as in the varlen API of section 3.7.6.

Readings taken where the pages are silent:

* soft-cap acts on the *scaled* score: s <- c * tanh(s / c) with s = scale * q.k;
* causal means kv <= q (diagonal visible); the sliding window is one-sided and causal:
  visible iff 0 <= q - kv <= window; the symmetric window (mask kind 4) is
  visible iff |q - kv| <= window, with no causality;
* the ALiBi bias of query head h is -slope_h * |q - kv| (natural-log units, the slopes
  given per query head), added after the soft-cap and before the mask;
* the document mask is "same document AND kv <= q", the documents given by int32
  boundaries [0, ..., Nk] shared by every batch entry;
* masks other than "none" need Nq == Nk;
* a row with no visible key has O = 0 and LSE = -inf;
* the log-sum-exp is the natural logarithm;
* KV head of query head h is h // (Hq // Hkv).

Precision: every value is converted to float64 before any arithmetic; S and P are
materialised for a block of query rows against *all* keys (no blocking along the key
axis in the plain definition).
"""
from __future__ import annotations

import math

import numpy as np

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_SLIDING_CAUSAL = 2
MASK_DOCUMENT_CAUSAL = 3
MASK_SLIDING = 4

TILE_EMPTY = 0
TILE_PARTIAL = 1
TILE_FULL = 2


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def default_scale(d: int) -> float:
    """softmax_scale=None means 1/sqrt(d): FlashAttention page, "flash-attn 라이브러리 직접
    사용" (``softmax_scale=None``) and "PyTorch SDPA를 통한 FlashAttention 사용"
    (``scale=None``)."""
    return 1.0 / math.sqrt(d)


def document_ids(idx, doc_offsets) -> np.ndarray:
    """Document index of each token position, from cumulative boundaries
    [0, L_0, L_0+L_1, ..., N] ("3.7 어텐션 II", section 3.7.6, ``cu_seqlens``)."""
    offs = np.asarray(doc_offsets, dtype=np.int64)
    return np.searchsorted(offs, np.asarray(idx, dtype=np.int64), side="right") - 1


def visible(q_idx, kv_idx, mask_kind: int, window: int = 0, doc_offsets=None) -> np.ndarray:
    """Boolean mask: True where query position q_idx may attend to key position kv_idx.

    Broadcasts q_idx against kv_idx.  Definitions: causal = "self and earlier tokens"
    ("Attention 최적화가 어려운 이유", "Attention의 계산 흐름"); sliding window = the
    FlexAttention page's ``|q_idx - kv_idx| <= window`` combined with causality; document
    = both positions inside the same packed sequence ("3.7 어텐션 II", 3.7.6), causal
    inside it.
    """
    q = np.asarray(q_idx, dtype=np.int64)
    kv = np.asarray(kv_idx, dtype=np.int64)
    if mask_kind == MASK_NONE:
        return np.ones(np.broadcast(q, kv).shape, dtype=bool)
    if mask_kind == MASK_SLIDING:
        return np.abs(q - kv) <= window
    causal = kv <= q
    if mask_kind == MASK_CAUSAL:
        return causal
    if mask_kind == MASK_SLIDING_CAUSAL:
        return causal & (np.abs(q - kv) <= window)
    if mask_kind == MASK_DOCUMENT_CAUSAL:
        if doc_offsets is None:
            raise ValueError("document mask needs doc_offsets")
        return causal & (document_ids(q, doc_offsets) == document_ids(kv, doc_offsets))
    raise ValueError(f"unknown mask kind {mask_kind}")


def softcap_scores(s: np.ndarray, softcap: float) -> np.ndarray:
    """tanh soft-capping of a score: c * tanh(s / c); c <= 0 means no cap (reading c1)."""
    if softcap and softcap > 0:
        return softcap * np.tanh(s / softcap)
    return s


def head_scores(q_rows, K, scale: float, softcap: float, row_idx, mask_kind: int,
                window: int, doc_offsets, kv_idx=None, alibi_slope: float = 0.0) -> np.ndarray:
    """Materialised score block S (rows x keys), -inf where masked.

    S = scale * Q K^T, then the score hook (soft-cap), then the ALiBi distance bias, then
    the mask: FlexAttention page section 2 (the hook sees the score right after Q.K^T);
    "3.7 어텐션 II" 3.7.5 (bias added before the softmax); the standard_attention listing
    on the FlashAttention page (masked_fill with -inf)."""
    Q = _f64(q_rows)
    Kf = _f64(K)
    S = scale * (Q @ Kf.T)
    S = softcap_scores(S, softcap)
    if kv_idx is None:
        kv_idx = np.arange(Kf.shape[0])
    if alibi_slope:
        dist = np.abs(np.asarray(row_idx, dtype=np.float64)[:, None]
                      - np.asarray(kv_idx, dtype=np.float64)[None, :])
        S = S - float(alibi_slope) * dist
    vis = visible(np.asarray(row_idx)[:, None], np.asarray(kv_idx)[None, :],
                  mask_kind, window, doc_offsets)
    return np.where(vis, S, -np.inf)


def softmax_rows(S: np.ndarray):
    """Row softmax of a score block with -inf entries.

    Returns (P, m, l) with P = exp(S - m) / l, m = row max, l = sum exp(S - m).  A row
    whose entries are all -inf gets P = 0, m = -inf, l = 0 (reading c6)."""
    m = S.max(axis=1)
    safe_m = np.where(np.isfinite(m), m, 0.0)
    E = np.exp(S - safe_m[:, None])          # exp(-inf) == 0 exactly
    l = E.sum(axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        P = np.where(l[:, None] > 0, E / np.where(l > 0, l, 1.0)[:, None], 0.0)
    return P, m, l


def attention_head(q_rows, row_idx, K, V, scale: float, mask_kind: int = MASK_NONE,
                   window: int = 0, softcap: float = 0.0, doc_offsets=None,
                   return_probs: bool = False, kv_idx=None, alibi_slope: float = 0.0):
    """Exact attention for some query rows of one (batch, head) against all keys.

    O_i = sum_j P_ij V_j and LSE_i = m_i + ln(l_i) ("어텐션 최적화" Step 3;
    FlashAttention page "Recomputation 전략" for the saved m, l)."""
    S = head_scores(q_rows, K, scale, softcap, row_idx, mask_kind, window, doc_offsets,
                    kv_idx=kv_idx, alibi_slope=alibi_slope)
    P, m, l = softmax_rows(S)
    O = P @ _f64(V)
    with np.errstate(divide="ignore"):
        lse = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    if return_probs:
        return O, lse, P
    return O, lse


def attention(q, k, v, scale=None, mask_kind: int = MASK_NONE, window: int = 0,
              softcap: float = 0.0, doc_offsets=None, row_chunk: int = 256, alibi_slopes=None):
    """Full oracle: q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] (any real dtype) -> (O, LSE) in fp64.

    O is [B,Hq,Nq,dv], LSE is [B,Hq,Nq].  Query head h reads KV head h // (Hq // Hkv);
    ``alibi_slopes`` (length Hq, or None) gives head h the bias -slope_h * |q - kv|."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if mask_kind != MASK_NONE and Nq != Nk:
        raise ValueError("masks need Nq == Nk")
    G = Hq // Hkv
    if scale is None or scale <= 0:
        scale = default_scale(d)
    O = np.zeros((B, Hq, Nq, v.shape[3]))
    lse = np.zeros((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            for r0 in range(0, Nq, row_chunk):
                rows = np.arange(r0, min(Nq, r0 + row_chunk))
                O[b, h, rows], lse[b, h, rows] = attention_head(
                    q[b, h, rows], rows, k[b, hk], v[b, hk], scale, mask_kind, window,
                    softcap, doc_offsets,
                    alibi_slope=0.0 if alibi_slopes is None else float(alibi_slopes[h]))
    return O, lse


def attention_backward(q, k, v, dout, scale=None, mask_kind: int = MASK_NONE, window: int = 0,
                       softcap: float = 0.0, doc_offsets=None, alibi_slopes=None,
                       row_chunk: int = 256):
    """Gradients (dQ, dK, dV) in fp64 of L with dL/dO = dout, for O = attention(q, k, v, ...).

    The pages fix *how* the backward pass is organised -- S and P recomputed from the saved
    row statistics instead of an N x N matrix kept from the forward pass (FlashAttention
    page, "Recomputation 전략" and "FlashAttention v1: Tiling + Recomputation") -- and the
    gradients are the calculus of the definition, written out per block of query rows:
      dV = P^T dO;  dP = dO V^T;  D_i = sum_j P_ij dP_ij = dO_i . O_i;
      dS = P * (dP - D)  (the softmax Jacobian);  with a soft-cap the score s = c tanh(x / c)
      of the scaled product x contributes dx = dS (1 - tanh^2(x / c));
      dQ = scale dX K;  dK = scale dX^T Q  (X = scale Q K^T; the ALiBi bias and the mask do
      not depend on q, k, v).  A KV head's dK, dV sum over its query-head group.
    Masked entries have P = 0 and so contribute nothing; rows with no visible key give 0."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    dout = _f64(dout)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    if scale is None or scale <= 0:
        scale = default_scale(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            slope = 0.0 if alibi_slopes is None else float(alibi_slopes[h])
            for r0 in range(0, Nq, row_chunk):
                rows = np.arange(r0, min(Nq, r0 + row_chunk))
                S = head_scores(q[b, h, rows], k[b, hk], scale, softcap, rows, mask_kind,
                                window, doc_offsets, alibi_slope=slope)
                P, _, _ = softmax_rows(S)
                O = P @ v[b, hk]
                dO = dout[b, h, rows]
                dP = dO @ v[b, hk].T
                D = (dO * O).sum(axis=1)
                dS = P * (dP - D[:, None])
                if softcap and softcap > 0:
                    X = scale * (q[b, h, rows] @ k[b, hk].T)
                    dS = dS * (1.0 - np.tanh(X / softcap) ** 2)
                dq[b, h, rows] = scale * (dS @ k[b, hk])
                dk[b, hk] += scale * (dS.T @ q[b, h, rows])
                dv[b, hk] += P.T @ dO
    return dq, dk, dv


def attention_tiled_online(q, k, v, scale=None, block_q: int = 2, block_kv: int = 3,
                           mask_kind: int = MASK_NONE, window: int = 0,
                           softcap: float = 0.0, doc_offsets=None, alibi_slopes=None):
    """The blockwise online-softmax form of the FlashAttention page ("Online Softmax와 블록
    단위 누적", "알고리즘 의사코드"), kept in its normalised-O form.

    For each query block and each key block j, in order:
      m_loc = rowmax(S_j); P_loc = exp(S_j - m_loc); l_loc = rowsum(P_loc)
      m_new = max(m, m_loc); alpha = exp(m - m_new); beta = exp(m_loc - m_new)
      l_new = alpha * l + beta * l_loc
      O     = (alpha * l * O + beta * P_loc V_j) / l_new
    Rows that have seen no visible key yet keep m = -inf, l = 0, O = 0 (reading c6, which
    the listing leaves undefined).  Used only to check the plain oracle."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    if scale is None or scale <= 0:
        scale = default_scale(d)
    O = np.zeros((B, Hq, Nq, v.shape[3]))
    M = np.full((B, Hq, Nq), -np.inf)
    L = np.zeros((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            for i0 in range(0, Nq, block_q):
                rows = np.arange(i0, min(Nq, i0 + block_q))
                m = np.full(len(rows), -np.inf)
                l = np.zeros(len(rows))
                o = np.zeros((len(rows), v.shape[3]))
                for j0 in range(0, Nk, block_kv):
                    cols = np.arange(j0, min(Nk, j0 + block_kv))
                    S = head_scores(q[b, h, rows], k[b, hk, cols], scale, softcap, rows,
                                    mask_kind, window, doc_offsets, kv_idx=cols,
                                    alibi_slope=0.0 if alibi_slopes is None
                                    else float(alibi_slopes[h]))
                    m_loc = S.max(axis=1)
                    has = np.isfinite(m_loc)
                    P_loc = np.where(has[:, None],
                                     np.exp(S - np.where(has, m_loc, 0.0)[:, None]), 0.0)
                    l_loc = P_loc.sum(axis=1)
                    m_new = np.maximum(m, m_loc)
                    live = np.isfinite(m_new)
                    alpha = np.where(np.isfinite(m), np.exp(m - np.where(live, m_new, 0.0)), 0.0)
                    beta = np.where(has, np.exp(m_loc - np.where(live, m_new, 0.0)), 0.0)
                    l_new = alpha * l + beta * l_loc
                    pv = P_loc @ v[b, hk, cols]
                    num = (alpha * l)[:, None] * o + beta[:, None] * pv
                    o = np.where(live[:, None], num / np.where(l_new > 0, l_new, 1.0)[:, None], 0.0)
                    m, l = m_new, l_new
                O[b, h, rows] = o
                M[b, h, rows] = m
                L[b, h, rows] = l
    with np.errstate(divide="ignore"):
        lse = np.where(L > 0, M + np.log(np.where(L > 0, L, 1.0)), -np.inf)
    return O, lse


def merge_partials(o_parts, lse_parts):
    """Combine per-split partial results by the rescaling recurrence ("3.7 어텐션 II",
    3.7.4: the splits' maxima and sums are re-normalised and combined).

    o_parts [..., S, dv] (each split normalised by its own sum), lse_parts [..., S]:
      L = max_s LSE_s; w_s = exp(LSE_s - L); O = sum_s w_s O_s / sum_s w_s;
      LSE = L + ln(sum_s w_s).  Splits with LSE = -inf carry weight 0."""
    o_parts = _f64(o_parts)
    lse_parts = _f64(lse_parts)
    Lmax = lse_parts.max(axis=-1)
    live = np.isfinite(Lmax)
    w = np.where(np.isfinite(lse_parts),
                 np.exp(lse_parts - np.where(live, Lmax, 0.0)[..., None]), 0.0)
    wsum = w.sum(axis=-1)
    with np.errstate(invalid="ignore", divide="ignore"):
        O = np.where(live[..., None],
                     (w[..., None] * o_parts).sum(axis=-2) / np.where(wsum > 0, wsum, 1.0)[..., None],
                     0.0)
        lse = np.where(live, Lmax + np.log(np.where(wsum > 0, wsum, 1.0)), -np.inf)
    return O, lse


def split_bounds(T: int, num_splits: int, tile: int = 1):
    """Split of T keys into num_splits contiguous slices that cut only at multiples of
    `tile` (the last slice ends at T): slice s holds tiles [s n / S, (s + 1) n / S) of the
    n = ceil(T / tile) tiles, so sizes differ by at most one tile (tile = 1: an even split of
    the keys).  Which slices FlashDecoding uses is free; merging is exact for any of them."""
    n = -(-T // tile)
    return [(min(T, (s * n // num_splits) * tile), min(T, ((s + 1) * n // num_splits) * tile))
            for s in range(num_splits)]


def decode_splitkv(q, k_cache, v_cache, num_splits: int, scale=None, tile: int = 1):
    """FlashDecoding reference ("3.7 어텐션 II", 3.7.4): q [B,Hq,1,d] against a
    contiguous cache [B,Hkv,T,d]; every split is attended separately (plain definition on
    its slice) and the partials are merged with ``merge_partials``.

    Returns (O [B,Hq,1,dv], LSE [B,Hq,1], O_parts [B,Hq,S,dv], LSE_parts [B,Hq,S])."""
    q = _f64(q)
    k_cache = _f64(k_cache)
    v_cache = _f64(v_cache)
    B, Hq, Nq, d = q.shape
    T = k_cache.shape[2]
    if scale is None or scale <= 0:
        scale = default_scale(d)
    G = Hq // k_cache.shape[1]
    S = num_splits
    o_parts = np.zeros((B, Hq, Nq, S, v_cache.shape[3]))
    lse_parts = np.full((B, Hq, Nq, S), -np.inf)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            for s, (t0, t1) in enumerate(split_bounds(T, S, tile)):
                if t1 <= t0:
                    continue
                o, l = attention_head(q[b, h], np.arange(Nq), k_cache[b, hk, t0:t1],
                                      v_cache[b, hk, t0:t1], scale)
                o_parts[b, h, :, s] = o
                lse_parts[b, h, :, s] = l
    O, lse = merge_partials(o_parts, lse_parts)
    return O, lse, o_parts, lse_parts


def gather_paged(pages, block_table_row, length: int):
    """The first ``length`` cache rows of one sequence from a paged cache: pages
    [num_pages, Hkv, page_size, d], the sequence's logical page j is physical page
    block_table_row[j] (PagedAttention's page table, "3.7 어텐션 II", 3.7.4 and 3.7.8).
    Returns [Hkv, length, d]."""
    pages = _f64(pages)
    page_size = pages.shape[2]
    n = -(-length // page_size) if length > 0 else 0
    if n == 0:
        return np.zeros((pages.shape[1], 0, pages.shape[3]))
    rows = np.concatenate([pages[int(block_table_row[j])] for j in range(n)], axis=1)
    return rows[:, :length]


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale=None):
    """Decode attention over paged, variable-length caches: query row (b, h) attends to
    the seq_lens[b] cache rows of sequence b gathered through its page table (plain
    definition on the gathered keys; every key visible).  q [B,Hq,1,d].
    Returns (O [B,Hq,1,dv], LSE [B,Hq,1]); a sequence of length 0 gives O = 0, LSE = -inf."""
    q = _f64(q)
    B, Hq, Nq, d = q.shape
    Hkv = np.asarray(k_pages).shape[1]
    G = Hq // Hkv
    if scale is None or scale <= 0:
        scale = default_scale(d)
    O = np.zeros((B, Hq, Nq, np.asarray(v_pages).shape[3]))
    lse = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        T = int(seq_lens[b])
        if T == 0:
            continue
        K = gather_paged(k_pages, block_table[b], T)
        V = gather_paged(v_pages, block_table[b], T)
        for h in range(Hq):
            O[b, h], lse[b, h] = attention_head(q[b, h], np.arange(Nq), K[h // G], V[h // G],
                                                scale)
    return O, lse


def tile_map(B: int, Nq: int, Nk: int, mask_kind: int, window: int = 0, doc_offsets=None,
             block_q: int = 128, block_kv: int = 128) -> np.ndarray:
    """Block-sparsity map at 128x128 granularity (FlexAttention page, section 2, item on
    BlockMask / early-out), by brute force over every element of every tile.

    map[b, i, j] = 0 if no (q, kv) pair of tile (i, j) is visible, 2 if every pair is,
    1 otherwise.  Only positions q < Nq, kv < Nk are pairs.  The mask is the same for
    every batch entry."""
    nqt = -(-Nq // block_q)
    nkt = -(-Nk // block_kv)
    out = np.zeros((B, nqt, nkt), dtype=np.uint8)
    cols = np.arange(Nk)
    for i in range(nqt):
        rows = np.arange(i * block_q, min(Nq, (i + 1) * block_q))
        vis = visible(rows[:, None], cols[None, :], mask_kind, window, doc_offsets)
        for j in range(nkt):
            blk = vis[:, j * block_kv: min(Nk, (j + 1) * block_kv)]
            if blk.all():
                out[:, i, j] = TILE_FULL
            elif blk.any():
                out[:, i, j] = TILE_PARTIAL
    return out


def visible_pairs(Nq: int, Nk: int, mask_kind: int, window: int = 0, doc_offsets=None,
                  row_chunk: int = 1024) -> int:
    """Number of visible (q, kv) pairs of one head, counted element by element."""
    total = 0
    cols = np.arange(Nk)
    for r0 in range(0, Nq, row_chunk):
        rows = np.arange(r0, min(Nq, r0 + row_chunk))
        total += int(visible(rows[:, None], cols[None, :], mask_kind, window, doc_offsets).sum())
    return total
