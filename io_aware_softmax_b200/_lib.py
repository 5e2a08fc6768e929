"""ctypes loader for ``libattn_b200.so`` and the C-ABI signatures of ``include/attn.h``.

There is no fallback: if the shared library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libattn_b200.so")

c_int, c_float, c_void_p, c_size_t, c_longlong = (ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                                  ctypes.c_size_t, ctypes.c_longlong)
c_int_p = ctypes.POINTER(ctypes.c_int)
c_float_p = ctypes.POINTER(ctypes.c_float)

# name -> (restype, argtypes), in the order of include/attn.h
SIGNATURES = {
    "attn_fwd": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                         c_int, c_int, c_int, c_float, c_int, c_int, c_float, c_void_p, c_int,
                         c_void_p]),
    "attn_fwd_alibi": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                               c_int, c_int, c_int, c_int, c_float, c_int, c_int, c_float,
                               c_void_p, c_int, c_void_p, c_void_p]),
    "attn_decode_paged": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                  c_float, c_int, c_void_p, c_size_t, c_void_p]),
    "attn_bwd_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "attn_bwd": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                         c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_float,
                         c_int, c_int, c_float, c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "attn_bwd_alibi": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                               c_int, c_float, c_int, c_int, c_float, c_void_p, c_int, c_void_p,
                               c_void_p, c_size_t, c_void_p]),
    "attn_quantize_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                  c_int, c_int, c_int, c_void_p, c_void_p]),
    "attn_fwd_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                             c_float, c_int, c_int, c_void_p, c_int, c_void_p]),
    "attn_blockmap": (c_int, [c_int, c_int, c_int, c_int, c_int, c_void_p, c_int, c_void_p,
                              c_void_p]),
    "attn_decode_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "attn_decode_default_splits": (c_int, [c_int, c_int, c_int, c_int]),
    "attn_decode_splitkv": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                    c_int, c_int, c_int, c_int, c_float, c_int, c_void_p,
                                    c_size_t, c_void_p]),
    "attn_decode_splitkv_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_int, c_int, c_int, c_int, c_int, c_float, c_int,
                                            c_void_p]),
    "attn_decode_merge": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_longlong, c_int,
                                  c_int, c_void_p]),
    "attn_get_device_status": (c_int, [c_void_p]),
    "attn_last_error_site": (c_int, []),
    "attn_set_wait_limit_ns": (c_int, [ctypes.c_ulonglong]),
    "attn_status_string": (ctypes.c_char_p, [c_int]),
    "attn_version": (c_int, []),
}

_lock = threading.Lock()
_lib = None


class LibraryMissing(RuntimeError):
    pass


def load(path: str = LIB_PATH):
    """Loads the library once and attaches the signatures; raises LibraryMissing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise LibraryMissing(
                f"{path} is missing: build it with `python -m io_aware_softmax_b200.build` "
                "(there is no non-CUDA implementation to fall back to)")
        try:
            lib = ctypes.CDLL(path)
        except OSError as e:
            raise LibraryMissing(f"cannot load {path}: {e}") from e
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib
