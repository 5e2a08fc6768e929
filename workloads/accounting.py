"""Work and byte accounting for the benchmark (closed forms, integer arithmetic).

Useful FLOPs of exact attention count only visible (query, key) pairs: each costs d
multiply-adds for Q.K and d for P.V, i.e. 4*d flops.  Decode moves the whole K and V
cache once per step.  These counts are checked against element-by-element counts of the
oracle's mask in the CPU tests.
"""
from __future__ import annotations

from . import MASK_CAUSAL, MASK_DOCUMENT_CAUSAL, MASK_NONE, MASK_SLIDING, MASK_SLIDING_CAUSAL


def visible_pairs(Nq: int, Nk: int, mask_kind: int, window: int = 0, doc_offsets=None) -> int:
    """Visible pairs of one head for each mask kind, in closed form."""
    if mask_kind == MASK_NONE:
        return Nq * Nk
    N = Nq
    if mask_kind == MASK_CAUSAL:
        return N * (N + 1) // 2
    if mask_kind == MASK_SLIDING_CAUSAL:
        n1 = min(N, window)
        return n1 * (n1 + 1) // 2 + (N - n1) * (window + 1)
    if mask_kind == MASK_SLIDING:
        # row i sees [max(0, i - w), min(N - 1, i + w)]: N (2w + 1) minus the parts cut off
        # at both ends, w - i keys for each of the first min(N, w) rows (and symmetrically)
        w = window
        n1 = min(N, w)
        cut = n1 * w - n1 * (n1 - 1) // 2
        return N * (2 * w + 1) - 2 * cut
    if mask_kind == MASK_DOCUMENT_CAUSAL:
        offs = [int(x) for x in doc_offsets]
        return sum((e - s) * (e - s + 1) // 2 for s, e in zip(offs[:-1], offs[1:]))
    raise ValueError(mask_kind)


def prefill_useful_flops(B: int, Hq: int, Nq: int, Nk: int, d: int, mask_kind: int,
                         window: int = 0, doc_offsets=None) -> int:
    return 4 * d * visible_pairs(Nq, Nk, mask_kind, window, doc_offsets) * B * Hq


def _row_interval(q: int, Nk: int, mask_kind: int, window: int, doc_offsets) -> tuple:
    """Visible keys [lo, hi] of query row q (lo > hi: none); the intervals are non-decreasing
    in q at both ends for every mask kind."""
    last = Nk - 1
    if mask_kind == MASK_NONE:
        return 0, last
    if mask_kind == MASK_CAUSAL:
        return 0, min(q, last)
    if mask_kind == MASK_SLIDING_CAUSAL:
        return max(0, q - window), min(q, last)
    if mask_kind == MASK_SLIDING:
        return max(0, q - window), min(q + window, last)
    if mask_kind == MASK_DOCUMENT_CAUSAL:
        offs = [int(x) for x in doc_offsets]
        start = max([o for o in offs[:-1] if o <= q], default=0)
        return start, min(q, last)
    raise ValueError(mask_kind)


def executed_tiles(Nq: int, Nk: int, mask_kind: int, window: int = 0, doc_offsets=None,
                   tile: int = 128) -> int:
    """(query tile, key tile) pairs the prefill kernel runs for one head: each query tile
    walks the key tiles from its first row's first visible key to its last row's last one."""
    n = 0
    for q0 in range(0, Nq, tile):
        lo, _ = _row_interval(q0, Nk, mask_kind, window, doc_offsets)
        _, hi = _row_interval(min(q0 + tile, Nq) - 1, Nk, mask_kind, window, doc_offsets)
        if hi >= lo:
            n += hi // tile - lo // tile + 1
    return n


def prefill_executed_flops(B: int, Hq: int, Nq: int, Nk: int, d: int, mask_kind: int,
                           window: int = 0, doc_offsets=None, tile: int = 128) -> int:
    """FLOPs the tensor cores execute: full tile products for every executed tile pair."""
    return 4 * d * tile * tile * executed_tiles(Nq, Nk, mask_kind, window, doc_offsets,
                                                tile) * B * Hq


def backward_useful_flops(B: int, Hq: int, Nq: int, Nk: int, d: int, mask_kind: int,
                          window: int = 0, doc_offsets=None) -> int:
    """Useful FLOPs of the backward pass: five products per visible pair (S recomputed,
    dP = dO V^T, dV = P^T dO, dQ = dS K, dK = dS^T Q), 2 d flops each."""
    return 10 * d * visible_pairs(Nq, Nk, mask_kind, window, doc_offsets) * B * Hq


def decode_kv_bytes(B: int, Hkv: int, T: int, d: int, elem_bytes: int = 2) -> int:
    """Bytes of K plus V read by one decode step (each cache byte read once)."""
    return 2 * B * Hkv * T * d * elem_bytes


def decode_io_bytes(B: int, Hq: int, Hkv: int, T: int, d: int) -> int:
    """All HBM bytes a decode step must move: the KV cache, q (bf16), O (bf16), LSE (fp32)."""
    return decode_kv_bytes(B, Hkv, T, d) + B * Hq * d * 2 * 2 + B * Hq * 4


def kv_cache_bytes(Hkv: int, T: int, d: int, B: int = 1, elem_bytes: int = 2) -> int:
    """K+V cache size of one layer."""
    return 2 * B * Hkv * T * d * elem_bytes


def score_matrix_bytes(B: int, H: int, N: int, elem_bytes: int = 2) -> int:
    """Bytes of a materialised N x N score matrix for every (batch, head)."""
    return B * H * N * N * elem_bytes


def prefill_io_bytes(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int) -> int:
    """Compulsory HBM bytes of one prefill call: Q, K, V read once, O and LSE written."""
    return 2 * d * (B * Hq * Nq + 2 * B * Hkv * Nk) + 2 * B * Hq * Nq * d + 4 * B * Hq * Nq
