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
