"""Exact fused IO-aware attention for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libattn_b200.so`` (C ABI in ``include/attn.h``);
this package is its thin Python binding.  Importing it does not load the library; the first
call does, and raises if the library is missing -- there is no other implementation.

Every C entry point has a binding of the same name (``attn_decode_splitkv``,
``attn_quantize_fp8``, ...); the shorter names (``attn_decode``, ``quantize_fp8``, ...) are
the same functions.
"""
from .api import (  # noqa: F401
    MASKS, AttnError, attn_blockmap, attn_bwd, attn_bwd_alibi, attn_bwd_workspace_bytes,
    attn_decode, attn_decode_default_splits, attn_decode_merge, attn_decode_paged, attn_decode_splitkv,
    attn_decode_splitkv_noalloc, attn_decode_workspace_bytes, attn_fwd, attn_fwd_alibi,
    attn_fwd_fp8, attn_get_device_status, attn_last_error_site, attn_merge, attn_quantize_fp8,
    attn_set_wait_limit_ns, attn_status_string, attn_version, bwd_workspace_bytes, decode_workspace_bytes,
    default_splits, device_status, quantize_fp8,
)
from ._lib import LIB_PATH, LibraryMissing, load as load_library  # noqa: F401

__all__ = [
    # the C entry points, one binding each
    "attn_fwd", "attn_fwd_alibi", "attn_bwd", "attn_bwd_alibi", "attn_bwd_workspace_bytes",
    "attn_quantize_fp8", "attn_fwd_fp8", "attn_blockmap", "attn_decode_workspace_bytes", "attn_decode_default_splits",
    "attn_decode_splitkv", "attn_decode_splitkv_noalloc", "attn_decode_paged",
    "attn_decode_merge", "attn_get_device_status", "attn_last_error_site",
    "attn_set_wait_limit_ns", "attn_status_string",
    "attn_version",
    # shorter names for the same functions
    "attn_decode", "attn_merge", "quantize_fp8", "bwd_workspace_bytes", "decode_workspace_bytes",
    "default_splits", "device_status",
    # plumbing
    "AttnError", "LibraryMissing", "load_library", "MASKS", "LIB_PATH",
]
