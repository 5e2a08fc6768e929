"""Seeded synthetic workloads shared by the tests, the oracle checks and ``bench.py``.

This module holds shapes, seeds and random-number draws only -- none of the attention
arithmetic.  Both the CUDA path and the fp64 oracle take their inputs from here, and
from nowhere else.

The five workloads are the shapes the pages' attention variants are exercised on:
a tiny parity case, causal multi-head prefill, sliding-window GQA prefill, packed
documents with a tanh soft-cap, and split-KV decode against a long contiguous cache.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_SLIDING_CAUSAL = 2
MASK_DOCUMENT_CAUSAL = 3
MASK_SLIDING = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill" | "decode"
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    mask_kind: int = MASK_NONE
    window: int = 0
    softcap: float = 0.0
    input_std: float = 1.0
    docs: bool = False        # packed documents of seeded uniform length
    doc_len_lo: int = 512
    doc_len_hi: int = 4096
    doc_seed: int = 0
    alibi: bool = False       # geometric ALiBi slopes 2^(-8 (h + 1) / Hq)
    seed: int = 0
    # One rank's part of a workload split over several GPUs (see rank_part): batch entries
    # [b0, b0 + B) and KV heads [hk0, hk0 + Hkv) of a workload with full_Hkv KV heads
    # (0: all of them).  The inputs are the same numbers the whole workload draws there.
    b0: int = 0
    hk0: int = 0
    full_Hkv: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> dict:
        out = {"workload": self.name, "B": self.B, "Hq": self.Hq, "Hkv": self.Hkv,
               "Nq": self.Nq, "Nk": self.Nk, "d": self.d, "mask": MASK_NAMES[self.mask_kind]}
        if self.window:
            out["window"] = self.window
        if self.softcap:
            out["softcap"] = self.softcap
        if self.alibi:
            out["alibi_slopes"] = "2^(-8 (h + 1) / Hq)"
        if self.docs:
            out["doc_len_range"] = [self.doc_len_lo, self.doc_len_hi]
            out["doc_seed"] = self.doc_seed
        out["input_std"] = self.input_std
        out["seed"] = self.seed
        if self.b0 or self.hk0 or self.full_Hkv:
            out["part"] = {"batch": [self.b0, self.b0 + self.B],
                           "kv_heads": [self.hk0, self.hk0 + self.Hkv]}
        return out


MASK_NAMES = {MASK_NONE: "none", MASK_CAUSAL: "causal",
              MASK_SLIDING_CAUSAL: "sliding_causal", MASK_DOCUMENT_CAUSAL: "document_causal",
              MASK_SLIDING: "sliding"}

TINY = Workload("tiny_b1_h2_n128_d64", "prefill", 1, 2, 2, 128, 128, 64, seed=1001)
TINY_CAUSAL = dataclasses.replace(TINY, name="tiny_b1_h2_n128_d64_causal",
                                  mask_kind=MASK_CAUSAL)
CAUSAL_MHA = Workload("causal_mha_b8_h32_n4096_d128", "prefill", 8, 32, 32, 4096, 4096, 128,
                      mask_kind=MASK_CAUSAL, seed=1002)
SWA_GQA = Workload("swa_gqa_b4_hq32_hkv8_n16384_w1024_d128", "prefill", 4, 32, 8, 16384,
                   16384, 128, mask_kind=MASK_SLIDING_CAUSAL, window=1024, seed=1003)
DOC_SOFTCAP = Workload("doc_softcap_b1_h16_n32768_d128", "prefill", 1, 16, 16, 32768, 32768,
                       128, mask_kind=MASK_DOCUMENT_CAUSAL, softcap=50.0, input_std=2.0,
                       docs=True, seed=1004)
DECODE = Workload("decode_b64_hq32_hkv8_t32768_d128", "decode", 64, 32, 8, 1, 32768, 128,
                  seed=1005)
# Widening rows: the ALiBi bias on the causal MHA shapes, and the symmetric (non-causal)
# window on the sliding-window GQA shapes.
ALIBI_MHA = dataclasses.replace(CAUSAL_MHA, name="alibi_causal_mha_b8_h32_n4096_d128",
                                alibi=True, seed=1006)
SWA_SYM_GQA = dataclasses.replace(SWA_GQA, name="swa_sym_gqa_b4_hq32_hkv8_n16384_w1024_d128",
                                  mask_kind=MASK_SLIDING, seed=1007)


def alibi_slopes(H: int):
    """The geometric ALiBi slopes 2^(-8 (h + 1) / H), one per query head."""
    return [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]


def workload_alibi_slopes(w: "Workload"):
    """The slopes of the query heads ``w`` holds (a rank's part keeps the whole workload's)."""
    G = w.Hq // w.Hkv
    full = alibi_slopes((w.full_Hkv or w.Hkv) * G)
    return full[w.hk0 * G:w.hk0 * G + w.Hq]

ALL = [TINY, TINY_CAUSAL, CAUSAL_MHA, SWA_GQA, DOC_SOFTCAP, DECODE, ALIBI_MHA, SWA_SYM_GQA]
BY_NAME = {w.name: w for w in ALL}


def doc_lengths(total: int, lo: int = 512, hi: int = 4096, seed: int = 0) -> list:
    """Document lengths drawn uniformly from [lo, hi] (inclusive) until they cover
    ``total`` tokens; the last one is truncated so that they sum to exactly ``total``."""
    rng = np.random.default_rng(seed)
    out = []
    acc = 0
    while acc < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - acc)
        out.append(n)
        acc += n
    return out


def doc_offsets_for(total: int, lo: int = 512, hi: int = 4096, seed: int = 0) -> np.ndarray:
    """Cumulative int32 boundaries [0, L0, L0+L1, ..., total] of ``doc_lengths``."""
    lens = doc_lengths(total, lo, hi, seed)
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def workload_doc_offsets(w: Workload) -> Optional[np.ndarray]:
    if not w.docs:
        return None
    return doc_offsets_for(w.Nk, w.doc_len_lo, w.doc_len_hi, w.doc_seed)


def _tensor_seed(seed: int, tensor_id: int, b: int) -> int:
    return ((seed * 16 + tensor_id) * 65536 + b) & 0x7FFFFFFFFFFFFFFF


def randn_bf16(shape, seed: int, tensor_id: int, std: float = 1.0, device="cpu", b0: int = 0):
    """bf16 tensor of i.i.d. N(0, std^2) draws: fp32 normal draws from a torch generator
    seeded per (seed, tensor, leading index), times ``std``, rounded to bf16 (RNE).

    The bits depend on ``device`` (CPU and CUDA generators differ) but are reproducible
    for a given device.  Drawing one leading slice at a time keeps the fp32 temporary
    small for multi-GiB caches.  ``b0`` draws leading slices b0, b0 + 1, ... (one rank's
    batch entries of a larger tensor)."""
    import torch

    out = torch.empty(tuple(shape), dtype=torch.bfloat16, device=device)
    g = torch.Generator(device=device)
    for b in range(shape[0]):
        g.manual_seed(_tensor_seed(seed, tensor_id, b0 + b))
        x = torch.randn(tuple(shape[1:]), generator=g, dtype=torch.float32, device=device)
        if std != 1.0:
            x.mul_(std)
        out[b].copy_(x)
        del x
    return out


def make_inputs(w: Workload, device="cpu"):
    """(q, k, v) bf16 tensors of workload ``w``: q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d].  For a
    rank's part, the part's slices of the whole workload's tensors."""
    G = w.Hq // w.Hkv if w.Hkv else 1
    hkv = w.full_Hkv or w.Hkv
    q = randn_bf16((w.B, hkv * G, w.Nq, w.d), w.seed, 0, w.input_std, device, w.b0)
    k = randn_bf16((w.B, hkv, w.Nk, w.d), w.seed, 1, w.input_std, device, w.b0)
    v = randn_bf16((w.B, hkv, w.Nk, w.d), w.seed, 2, w.input_std, device, w.b0)
    if hkv != w.Hkv:
        q = q[:, w.hk0 * G:(w.hk0 + w.Hkv) * G].contiguous()
        k = k[:, w.hk0:w.hk0 + w.Hkv].contiguous()
        v = v[:, w.hk0:w.hk0 + w.Hkv].contiguous()
    return q, k, v


def rank_part(w: Workload, world: int, rank: int) -> Workload:
    """The part of ``w`` that rank ``rank`` of ``world`` GPUs runs.  (batch, head) units are
    independent, so the ranks split them with no exchange: whole batch entries when
    ``world`` divides B, else whole KV-head groups (their query heads with them) when it
    divides Hkv; if neither, every rank runs the whole workload (replicas)."""
    if world <= 1:
        return w
    if w.B % world == 0:
        n = w.B // world
        return dataclasses.replace(w, B=n, b0=rank * n, full_Hkv=w.Hkv)
    if w.Hkv % world == 0:
        n = w.Hkv // world
        G = w.Hq // w.Hkv
        return dataclasses.replace(w, Hq=n * G, Hkv=n, hk0=rank * n, full_Hkv=w.Hkv)
    return w
