"""FP8 (E4M3) inputs for the attention oracle -- TEST INFRASTRUCTURE ONLY (see attention.py).

"FlashAttention 논문 분석: IO-Aware Exact Attention", section "FP8 지원과 정확도 유지", names
the two measures that keep FP8 attention accurate:

* block quantization: every block of rows gets its own scale, so each block uses the whole
  E4M3 range (here: scale = amax / 448, the largest finite E4M3 magnitude, per block of
  `block_rows` rows of one (batch, head));
* incoherent processing: Q and K are multiplied by a random orthogonal matrix before they
  are quantized, which spreads outliers over all columns; (Q M)(K M)^T = Q K^T, so the
  scores are unchanged.  The matrix here is M = diag(signs) H / sqrt(d), H the Sylvester
  Hadamard matrix (d a power of two) and signs a seeded +-1 vector.

What the FP8 path computes is then exact attention on the dequantized values (code times
block scale); ``attention_fp8`` is that, on top of the plain oracle.  The rounding of a
value to E4M3 is torch's float8_e4m3fn conversion (round to nearest even).
"""
from __future__ import annotations

import numpy as np
import torch

from .attention import _f64, attention

E4M3_MAX = 448.0


def hadamard(d: int) -> np.ndarray:
    """Sylvester's construction: H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def rotate(x, signs) -> np.ndarray:
    """x (..., d) times diag(signs) H / sqrt(d): an orthogonal map of the last axis."""
    x = _f64(x)
    d = x.shape[-1]
    return (x * _f64(signs)) @ hadamard(d) / np.sqrt(d)


def to_e4m3(x) -> np.ndarray:
    """Values rounded to the E4M3 grid (as float64), via torch's float8_e4m3fn conversion."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def quantize_blocks(x, block_rows: int):
    """Block quantization of x [B, H, N, d] (float32 arithmetic, as a kernel does it):
    per block of `block_rows` rows, scale = amax / 448 (1 for an all-zero block), codes =
    E4M3(x * (448 / amax)).  Returns (codes as float64 [B, H, N, d], scales [B, H, nblk])."""
    x32 = np.asarray(x, dtype=np.float32)
    B, H, N, d = x32.shape
    nblk = -(-N // block_rows)
    codes = np.zeros(x32.shape)
    scales = np.ones((B, H, nblk))
    for i in range(nblk):
        blk = x32[:, :, i * block_rows:(i + 1) * block_rows]
        amax = np.abs(blk).max(axis=(2, 3)).astype(np.float32)
        live = amax > 0
        inv = np.where(live, np.float32(E4M3_MAX) / np.where(live, amax, np.float32(1)),
                       np.float32(1)).astype(np.float32)
        codes[:, :, i * block_rows:(i + 1) * block_rows] = to_e4m3(blk * inv[:, :, None, None])
        scales[:, :, i] = np.where(live, amax.astype(np.float64) / E4M3_MAX, 1.0)
    return codes, scales


def dequantize_blocks(codes, scales, block_rows: int) -> np.ndarray:
    codes = _f64(codes)
    rep = np.repeat(_f64(scales), block_rows, axis=2)[:, :, : codes.shape[2]]
    return codes * rep[..., None]


def attention_fp8(q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, scale=None,
                  block_rows: int = 128, **kw):
    """Exact attention of the dequantized FP8 inputs: Q and K with per-block scales of
    `block_rows` rows, V [B, Hkv, Nk, d] with one scale per head (v_scales [B, Hkv])."""
    q = dequantize_blocks(q_codes, q_scales, block_rows)
    k = dequantize_blocks(k_codes, k_scales, block_rows)
    v = _f64(v_codes) * _f64(v_scales)[:, :, None, None]
    return attention(q, k, v, scale=scale, **kw)
