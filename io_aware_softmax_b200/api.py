"""Python binding of the C ABI: marshals torch tensors (device pointers, sizes, the current
CUDA stream) into the ``libattn_b200`` entry points.  Every step of the computation runs
in the library's CUDA kernels; nothing here computes attention.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import _lib

MASKS = {"none": 0, "causal": 1, "sliding_causal": 2, "document_causal": 3, "sliding": 4}

ATTN_OK = 0


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _lib.load()
        msg = lib.attn_status_string(status).decode()
        super().__init__(f"{where}: status {status} ({msg})")
        self.status = status


def _check(status: int, where: str):
    if status != ATTN_OK:
        raise AttnError(status, where)


def _mask_id(mask) -> int:
    if isinstance(mask, str):
        return MASKS[mask]
    return int(mask)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device, stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _on_gpu(t: torch.Tensor, name: str):
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, dims: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    _on_gpu(t, name)
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dimensions")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shape(t: torch.Tensor, name: str, shape):
    # the library reads and writes exactly the extents the sizes imply; a tensor of another
    # shape would let a kernel run past its allocation
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _same_device(ref: torch.Tensor, *named):
    for t, n in named:
        if t is not None and t.device != ref.device:
            raise ValueError(f"{n} is on {t.device}, the inputs on {ref.device}")


def _out(t: torch.Tensor, name: str, dtype: torch.dtype, shape, ref: torch.Tensor):
    """Checks a caller-supplied output tensor: dtype, exact shape, contiguous, ref's device."""
    _need(t, name, dtype, len(shape))
    _shape(t, name, shape)
    _same_device(ref, (t, name))


def _workspace(ws: torch.Tensor, ref: torch.Tensor) -> int:
    """Checks a caller-supplied workspace (any dtype) and returns its size in bytes."""
    if not isinstance(ws, torch.Tensor):
        raise TypeError("workspace must be a torch.Tensor")
    _on_gpu(ws, "workspace")
    if not ws.is_contiguous():
        raise ValueError("workspace must be contiguous")
    _same_device(ref, (ws, "workspace"))
    return ws.numel() * ws.element_size()


def _kv_shapes(k: torch.Tensor, v: torch.Tensor, B: int, d: int, kn: str, vn: str):
    if k.shape[0] != B or k.shape[3] != d:
        raise ValueError(f"{kn} {tuple(k.shape)} must have the batch {B} and head size {d} of q")
    _shape(v, vn, k.shape)


def _index(t: torch.Tensor) -> int:
    return t.device.index if t.device.index is not None else torch.cuda.current_device()


def _device(t: torch.Tensor):
    """Makes t's device current for the call: the library launches on the current device."""
    return torch.cuda.device(t.device)


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, scale: Optional[float] = None,
             mask="none", window: int = 0, softcap: float = 0.0,
             doc_offsets: Optional[torch.Tensor] = None, alibi_slopes: Optional[torch.Tensor] = None,
             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Fused prefill attention: q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] bf16 -> (O bf16, LSE fp32).

    ``alibi_slopes`` (fp32 [Hq] on the device) adds -slope_h * |q - kv| to the scores of
    query head h (attn_fwd_alibi)."""
    lib = _lib.load()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, 4)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    _kv_shapes(k, v, B, d, "k", "v")
    _same_device(q, (k, "k"), (v, "v"))
    if out is None:
        out = torch.empty_like(q)
    _out(out, "out", torch.bfloat16, (B, Hq, Nq, d), q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    _out(lse, "lse", torch.float32, (B, Hq, Nq), q)
    num_docs = 0
    if doc_offsets is not None:
        _need(doc_offsets, "doc_offsets", torch.int32, 1)
        _same_device(q, (doc_offsets, "doc_offsets"))
        num_docs = doc_offsets.numel() - 1
    with _device(q):
        if alibi_slopes is None:
            st = lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Nq, Nk,
                              d, float(scale or 0.0), _mask_id(mask), int(window),
                              float(softcap or 0.0), _ptr(doc_offsets), num_docs,
                              _stream(q.device, stream))
            _check(st, "attn_fwd")
        else:
            _need(alibi_slopes, "alibi_slopes", torch.float32, 1)
            _same_device(q, (alibi_slopes, "alibi_slopes"))
            if alibi_slopes.numel() != Hq:
                raise ValueError(f"alibi_slopes must hold Hq={Hq} slopes")
            st = lib.attn_fwd_alibi(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv,
                                    Nq, Nk, d, float(scale or 0.0), _mask_id(mask), int(window),
                                    float(softcap or 0.0), _ptr(doc_offsets), num_docs,
                                    _ptr(alibi_slopes), _stream(q.device, stream))
            _check(st, "attn_fwd_alibi")
    return out, lse


def bwd_workspace_bytes(B: int, Hq: int, Nq: int) -> int:
    return int(_lib.load().attn_bwd_workspace_bytes(B, Hq, Nq))


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
             lse: torch.Tensor, dout: torch.Tensor, *, scale: Optional[float] = None,
             mask="none", window: int = 0, doc_offsets: Optional[torch.Tensor] = None,
             dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
             dv: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
             alibi_slopes: Optional[torch.Tensor] = None, softcap: float = 0.0,
             stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Backward of attn_fwd: (dq, dk, dv) from q, k, v, attn_fwd's (o, lse) and dout.

    ``alibi_slopes`` (fp32 [Hq] on the device, as given to attn_fwd) selects attn_bwd_alibi;
    ``softcap`` is the soft-cap given to attn_fwd."""
    lib = _lib.load()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, n, torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if o.shape != q.shape or dout.shape != q.shape or tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("o and dout must have q's shape and lse [B, Hq, Nq]")
    _kv_shapes(k, v, B, d, "k", "v")
    _same_device(q, (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (lse, "lse"))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _out(dq, "dq", torch.bfloat16, q.shape, q)
    _out(dk, "dk", torch.bfloat16, k.shape, q)
    _out(dv, "dv", torch.bfloat16, k.shape, q)
    need = bwd_workspace_bytes(B, Hq, Nq)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace(workspace, q)
    num_docs = 0
    if doc_offsets is not None:
        _need(doc_offsets, "doc_offsets", torch.int32, 1)
        _same_device(q, (doc_offsets, "doc_offsets"))
        num_docs = doc_offsets.numel() - 1
    if alibi_slopes is not None:
        _need(alibi_slopes, "alibi_slopes", torch.float32, 1)
        _shape(alibi_slopes, "alibi_slopes", (Hq,))
        _same_device(q, (alibi_slopes, "alibi_slopes"))
    with _device(q):
        if alibi_slopes is None:
            st = lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                              _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, Nq, Nk, d,
                              float(scale or 0.0), _mask_id(mask), int(window), float(softcap or 0.0),
                              _ptr(doc_offsets), num_docs, _ptr(workspace), ws_bytes,
                              _stream(q.device, stream))
        else:
            st = lib.attn_bwd_alibi(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                    _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, Nq, Nk, d,
                                    float(scale or 0.0), _mask_id(mask), int(window), float(softcap or 0.0),
                                    _ptr(doc_offsets), num_docs, _ptr(alibi_slopes),
                                    _ptr(workspace), ws_bytes, _stream(q.device, stream))
    _check(st, "attn_bwd" if alibi_slopes is None else "attn_bwd_alibi")
    return dq, dk, dv


def quantize_fp8(x: torch.Tensor, *, block_rows: int = 128, transpose: bool = False,
                 n_pad: Optional[int] = None, signs: Optional[torch.Tensor] = None,
                 stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """E4M3 block quantization of x [B,H,N,d] bf16 -> (codes float8_e4m3fn, scales fp32
    [B,H,ceil(N/block_rows)]); codes are [B,H,N,d], or [B,H,d,n_pad] when transposed (V)."""
    lib = _lib.load()
    _need(x, "x", torch.bfloat16, 4)
    B, H, N, d = x.shape
    if int(block_rows) <= 0:
        raise ValueError("block_rows must be positive")
    if signs is not None:
        _need(signs, "signs", torch.float32, 1)
        _shape(signs, "signs", (d,))
        _same_device(x, (signs, "signs"))
    if transpose:
        n_pad = -(-N // 16) * 16 if n_pad is None else int(n_pad)
        out = torch.empty((B, H, d, n_pad), dtype=torch.float8_e4m3fn, device=x.device)
    else:
        n_pad = 0
        out = torch.empty((B, H, N, d), dtype=torch.float8_e4m3fn, device=x.device)
    scales = torch.empty((B, H, -(-N // block_rows)), dtype=torch.float32, device=x.device)
    with _device(x):
        st = lib.attn_quantize_fp8(_ptr(x), _ptr(out), _ptr(scales), B, H, N, d, int(block_rows),
                                   int(bool(transpose)), n_pad, _ptr(signs),
                                   _stream(x.device, stream))
    _check(st, "attn_quantize_fp8")
    return out, scales


def attn_fwd_fp8(q8: torch.Tensor, q_scales: torch.Tensor, k8: torch.Tensor,
                 k_scales: torch.Tensor, vt8: torch.Tensor, v_scales: torch.Tensor, *,
                 scale: Optional[float] = None, mask="none", window: int = 0,
                 doc_offsets: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, stream=None
                 ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Prefill on E4M3 inputs: q8 [B,Hq,Nq,d], k8 [B,Hkv,Nk,d], vt8 [B,Hkv,d,nk_pad] with
    per-block scales (q, k: [.., ceil(N/128)]) and per-head V scales [B,Hkv] -> (O, LSE)."""
    lib = _lib.load()
    for t, n in ((q8, "q8"), (k8, "k8"), (vt8, "vt8")):
        _need(t, n, torch.float8_e4m3fn, 4)
    B, Hq, Nq, d = q8.shape
    Hkv, Nk = k8.shape[1], k8.shape[2]
    nk_pad = vt8.shape[3]
    if k8.shape[0] != B or k8.shape[3] != d:
        raise ValueError(f"k8 {tuple(k8.shape)} must have the batch {B} and head size {d} of q8")
    if tuple(vt8.shape[:3]) != (B, Hkv, d):
        raise ValueError(f"vt8 {tuple(vt8.shape)} must be [B={B}, Hkv={Hkv}, d={d}, nk_pad]")
    for t, n, shape in ((q_scales, "q_scales", (B, Hq, -(-Nq // 128))),
                        (k_scales, "k_scales", (B, Hkv, -(-Nk // 128))),
                        (v_scales, "v_scales", (B, Hkv))):
        _need(t, n, torch.float32, len(shape))
        _shape(t, n, shape)
    _same_device(q8, (k8, "k8"), (vt8, "vt8"), (q_scales, "q_scales"), (k_scales, "k_scales"),
                 (v_scales, "v_scales"))
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=q8.device)
    _out(out, "out", torch.bfloat16, (B, Hq, Nq, d), q8)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q8.device)
    _out(lse, "lse", torch.float32, (B, Hq, Nq), q8)
    num_docs = 0
    if doc_offsets is not None:
        _need(doc_offsets, "doc_offsets", torch.int32, 1)
        _same_device(q8, (doc_offsets, "doc_offsets"))
        num_docs = doc_offsets.numel() - 1
    with _device(q8):
        st = lib.attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(q_scales), _ptr(k_scales),
                              _ptr(v_scales), _ptr(out), _ptr(lse), B, Hq, Hkv, Nq, Nk, nk_pad,
                              d, float(scale or 0.0), _mask_id(mask), int(window),
                              _ptr(doc_offsets), num_docs, _stream(q8.device, stream))
    _check(st, "attn_fwd_fp8")
    return out, lse


def attn_blockmap(B: int, Nq: int, Nk: int, *, mask="none", window: int = 0,
                  doc_offsets: Optional[torch.Tensor] = None, device=None,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """128x128 tile classes (0 empty, 1 partial, 2 full) as uint8 [B, ceil(Nq/128), ceil(Nk/128)]."""
    lib = _lib.load()
    if device is None:
        device = doc_offsets.device if doc_offsets is not None else torch.device("cuda")
    device = torch.device(device)
    shape = (B, -(-Nq // 128), -(-Nk // 128))
    if out is None:
        out = torch.empty(shape, dtype=torch.uint8, device=device)
    _out(out, "out", torch.uint8, shape, out)
    num_docs = 0
    if doc_offsets is not None:
        _need(doc_offsets, "doc_offsets", torch.int32, 1)
        _same_device(out, (doc_offsets, "doc_offsets"))
        num_docs = doc_offsets.numel() - 1
    with _device(out):
        st = lib.attn_blockmap(B, Nq, Nk, _mask_id(mask), int(window), _ptr(doc_offsets),
                               num_docs, _ptr(out), _stream(out.device, stream))
    _check(st, "attn_blockmap")
    return out


def decode_workspace_bytes(B: int, Hq: int, d: int, num_splits: int) -> int:
    return int(_lib.load().attn_decode_workspace_bytes(B, Hq, d, num_splits))


def default_splits(B: int, Hkv: int, T: int, device: int = 0) -> int:
    return int(_lib.load().attn_decode_default_splits(B, Hkv, T, device))


def attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, *,
                scale: Optional[float] = None, num_splits: Optional[int] = None,
                workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                lse: Optional[torch.Tensor] = None, stream=None
                ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split-KV decode: q [B,Hq,1,d], caches [B,Hkv,T,d] bf16 -> (O [B,Hq,1,d], LSE [B,Hq,1])."""
    lib = _lib.load()
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, n, torch.bfloat16, 4)
    B, Hq, nq, d = q.shape
    if nq != 1:
        raise ValueError("decode takes one query token per sequence")
    Hkv, T = k_cache.shape[1], k_cache.shape[2]
    _kv_shapes(k_cache, v_cache, B, d, "k_cache", "v_cache")
    _same_device(q, (k_cache, "k_cache"), (v_cache, "v_cache"))
    S = int(num_splits) if num_splits else default_splits(B, Hkv, T, _index(q))
    S = max(1, min(S, max(T, 1)))
    need = decode_workspace_bytes(B, Hq, d, S)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace(workspace, q)
    if out is None:
        out = torch.empty_like(q)
    _out(out, "out", torch.bfloat16, (B, Hq, 1, d), q)
    if lse is None:
        lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device)
    _out(lse, "lse", torch.float32, (B, Hq, 1), q)
    with _device(q):
        st = lib.attn_decode_splitkv(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
                                     B, Hq, Hkv, T, d, float(scale or 0.0), S, _ptr(workspace),
                                     ws_bytes, _stream(q.device, stream))
    _check(st, "attn_decode_splitkv")
    return out, lse


def attn_decode_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                      block_table: torch.Tensor, seq_lens: torch.Tensor, *,
                      scale: Optional[float] = None, num_splits: Optional[int] = None,
                      workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                      lse: Optional[torch.Tensor] = None, stream=None
                      ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split-KV decode over paged caches: q [B,Hq,1,d]; pages [num_pages,Hkv,page_size,d] bf16;
    block_table int32 [B, max_pages]; seq_lens int32 [B] -> (O [B,Hq,1,d], LSE [B,Hq,1])."""
    lib = _lib.load()
    _need(q, "q", torch.bfloat16, 4)
    for t, n in ((k_pages, "k_pages"), (v_pages, "v_pages")):
        _need(t, n, torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, nq, d = q.shape
    if nq != 1:
        raise ValueError("decode takes one query token per sequence")
    num_pages, Hkv, page_size = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    max_pages = block_table.shape[1]
    if block_table.shape[0] != B or seq_lens.numel() != B:
        raise ValueError("block_table and seq_lens need one row / entry per sequence")
    if k_pages.shape[3] != d:
        raise ValueError(f"k_pages {tuple(k_pages.shape)} must have the head size {d} of q")
    _shape(v_pages, "v_pages", k_pages.shape)
    _same_device(q, (k_pages, "k_pages"), (v_pages, "v_pages"), (block_table, "block_table"),
                 (seq_lens, "seq_lens"))
    t_cap = max_pages * page_size
    S = int(num_splits) if num_splits else default_splits(B, Hkv, max(t_cap, 1), _index(q))
    S = max(1, min(S, max(-(-t_cap // 64), 1)))
    need = decode_workspace_bytes(B, Hq, d, S)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace(workspace, q)
    if out is None:
        out = torch.empty_like(q)
    _out(out, "out", torch.bfloat16, (B, Hq, 1, d), q)
    if lse is None:
        lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device)
    _out(lse, "lse", torch.float32, (B, Hq, 1), q)
    with _device(q):
        st = lib.attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                   _ptr(seq_lens), _ptr(out), _ptr(lse), B, Hq, Hkv, num_pages,
                                   page_size, max_pages, d, float(scale or 0.0), S,
                                   _ptr(workspace), ws_bytes, _stream(q.device, stream))
    _check(st, "attn_decode_paged")
    return out, lse


def attn_merge(o_part: torch.Tensor, lse_part: torch.Tensor, *, out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Merge partials o_part fp32 [rows, S, d], lse_part fp32 [rows, S] -> (O bf16, LSE fp32)."""
    lib = _lib.load()
    _need(o_part, "o_part", torch.float32, 3)
    _need(lse_part, "lse_part", torch.float32, 2)
    rows, S, d = o_part.shape
    _shape(lse_part, "lse_part", (rows, S))
    _same_device(o_part, (lse_part, "lse_part"))
    if out is None:
        out = torch.empty((rows, d), dtype=torch.bfloat16, device=o_part.device)
    _out(out, "out", torch.bfloat16, (rows, d), o_part)
    if lse is None:
        lse = torch.empty((rows,), dtype=torch.float32, device=o_part.device)
    _out(lse, "lse", torch.float32, (rows,), o_part)
    with _device(o_part):
        st = lib.attn_decode_merge(_ptr(o_part), _ptr(lse_part), _ptr(out), _ptr(lse), rows, S,
                                   d, _stream(o_part.device, stream))
    _check(st, "attn_decode_merge")
    return out, lse


def device_status(stream=None, device=None) -> int:
    """Synchronises the stream and returns (and clears) the library's device error status."""
    lib = _lib.load()
    dev = torch.device(device) if device is not None else torch.device("cuda",
                                                                        torch.cuda.current_device())
    with torch.cuda.device(dev):
        return int(lib.attn_get_device_status(_stream(dev, stream)))


def attn_fwd_alibi(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   alibi_slopes: torch.Tensor, **kwargs) -> Tuple[torch.Tensor, torch.Tensor]:
    """attn_fwd with the ALiBi bias: query head h adds -alibi_slopes[h] * |q - kv|."""
    if alibi_slopes is None:
        raise ValueError("attn_fwd_alibi needs alibi_slopes (fp32 [Hq] on the device)")
    return attn_fwd(q, k, v, alibi_slopes=alibi_slopes, **kwargs)


def attn_bwd_alibi(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                   lse: torch.Tensor, dout: torch.Tensor, alibi_slopes: torch.Tensor,
                   **kwargs) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """attn_bwd for scores with the ALiBi bias of attn_fwd_alibi."""
    if alibi_slopes is None:
        raise ValueError("attn_bwd_alibi needs alibi_slopes (fp32 [Hq] on the device)")
    return attn_bwd(q, k, v, o, lse, dout, alibi_slopes=alibi_slopes, **kwargs)


def attn_decode_splitkv_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                *, scale: Optional[float] = None,
                                num_splits: Optional[int] = None,
                                out: Optional[torch.Tensor] = None,
                                lse: Optional[torch.Tensor] = None,
                                stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """attn_decode with the split partials in the library's own device array (no workspace;
    calls on one device share it, so issue them on one stream)."""
    lib = _lib.load()
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, n, torch.bfloat16, 4)
    B, Hq, nq, d = q.shape
    if nq != 1:
        raise ValueError("decode takes one query token per sequence")
    Hkv, T = k_cache.shape[1], k_cache.shape[2]
    _kv_shapes(k_cache, v_cache, B, d, "k_cache", "v_cache")
    _same_device(q, (k_cache, "k_cache"), (v_cache, "v_cache"))
    if out is None:
        out = torch.empty_like(q)
    _out(out, "out", torch.bfloat16, (B, Hq, 1, d), q)
    if lse is None:
        lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device)
    _out(lse, "lse", torch.float32, (B, Hq, 1), q)
    with _device(q):
        st = lib.attn_decode_splitkv_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out),
                                             _ptr(lse), B, Hq, Hkv, T, d, float(scale or 0.0),
                                             int(num_splits or 0), _stream(q.device, stream))
    _check(st, "attn_decode_splitkv_noalloc")
    return out, lse


def attn_status_string(status: int) -> str:
    return _lib.load().attn_status_string(int(status)).decode()


def attn_last_error_site() -> int:
    """Where the last bounded device wait that ran out gave up (0: none recorded)."""
    return int(_lib.load().attn_last_error_site())


def attn_set_wait_limit_ns(ns: int, device=None) -> None:
    """Limit of the kernels' pipeline waits on ``device`` (0: the built-in 0.5 s).  A wait
    that runs out makes the call report ATTN_ERR_DEVICE_TIMEOUT through device_status()."""
    lib = _lib.load()
    dev = torch.device(device) if device is not None else torch.device("cuda",
                                                                        torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(lib.attn_set_wait_limit_ns(int(ns)), "attn_set_wait_limit_ns")


def attn_version() -> int:
    return int(_lib.load().attn_version())


# Every C entry point of include/attn.h under its own name.
attn_decode_splitkv = attn_decode
attn_decode_merge = attn_merge
attn_quantize_fp8 = quantize_fp8
attn_get_device_status = device_status
attn_bwd_workspace_bytes = bwd_workspace_bytes
attn_decode_workspace_bytes = decode_workspace_bytes
attn_decode_default_splits = default_splits
