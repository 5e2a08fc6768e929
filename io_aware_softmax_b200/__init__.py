"""Exact fused IO-aware attention for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libattn_b200.so`` (C ABI in ``include/attn.h``);
this package is its thin Python binding.  Importing it does not load the library; the first
call does, and raises if the library is missing -- there is no other implementation.
"""
from .api import (  # noqa: F401
    MASKS, AttnError, attn_blockmap, attn_bwd, attn_decode, attn_decode_paged, attn_fwd,
    attn_fwd_fp8, attn_merge, bwd_workspace_bytes, decode_workspace_bytes, default_splits,
    device_status, quantize_fp8,
)
from ._lib import LIB_PATH, LibraryMissing, load as load_library  # noqa: F401

__all__ = ["attn_fwd", "attn_fwd_fp8", "quantize_fp8", "attn_bwd", "attn_blockmap", "attn_decode", "attn_decode_paged",
           "attn_merge", "bwd_workspace_bytes", "decode_workspace_bytes", "default_splits",
           "device_status", "AttnError", "LibraryMissing", "load_library", "MASKS", "LIB_PATH"]
