"""attn_decode_splitkv_noalloc: split-KV decode for callers that cannot allocate device memory.

Such callers (a plugin inside a host application that owns every device allocation, code
that must not allocate while a stream is captured into a CUDA graph, a loop with a fixed
memory budget) cannot hand attn_decode_splitkv a workspace.  The no-alloc entry point keeps
the split partials in a library-owned device array instead.  Here it is called through the
C ABI twice in a row (the second call finds the first call's partials still in the array)
and both results must equal the regular entry point's bit for bit: the two run the same
kernels on the same inputs and differ only in where the partials live.
This file is collected last so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import pytest
import torch

import workloads
from io_aware_softmax_b200 import _lib, attn_decode, device_status

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, kc, vc, o, lse, splits, scale=0.0):
    B, Hq, _, d = q.shape
    Hkv, T = kc.shape[1], kc.shape[2]
    stream = torch.cuda.current_stream().cuda_stream
    return lib.attn_decode_splitkv_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                           o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, T, d,
                                           ctypes.c_float(scale), splits, stream)


@pytest.mark.parametrize("B,Hq,Hkv,T,d,splits", [(4, 16, 4, 3000, 128, 7), (2, 8, 2, 777, 64, 0)])
def test_noalloc_matches_the_workspace_entry_point_twice(B, Hq, Hkv, T, d, splits):
    lib = _lib.load()
    torch.cuda.set_device(0)
    for call in range(2):
        seed = 900 + 10 * call + d
        q = workloads.randn_bf16((B, Hq, 1, d), seed, 0).cuda()
        kc = workloads.randn_bf16((B, Hkv, T, d), seed, 1).cuda()
        vc = workloads.randn_bf16((B, Hkv, T, d), seed, 2).cuda()
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
        st = _noalloc(lib, q, kc, vc, o, lse, splits)
        assert st == 0, lib.attn_status_string(st)
        o_ref, lse_ref = attn_decode(q, kc, vc, num_splits=splits or None)
        assert device_status() == 0
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref), f"no-alloc call {call}"


def test_noalloc_rejects_requests_beyond_its_array():
    lib = _lib.load()
    B, Hq, Hkv, T, d = 64, 32, 8, 256, 128
    splits = 64               # 64*32*64*129*4 bytes of partials > 32 MiB
    q = torch.zeros((B, Hq, 1, d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((B, Hkv, T, d), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.attn_decode_splitkv_noalloc(q.data_ptr(), kv.data_ptr(), kv.data_ptr(), o.data_ptr(),
                                         lse.data_ptr(), B, Hq, Hkv, T, d, ctypes.c_float(0.0),
                                         splits, stream)
    assert st == -6 and lib.attn_status_string(st) == b"workspace missing or too small"
    # an invalid request is reported as such, not as too large: 32 query heads over 6 KV
    # heads, with partials far beyond the array
    st = lib.attn_decode_splitkv_noalloc(q.data_ptr(), kv.data_ptr(), kv.data_ptr(), o.data_ptr(),
                                         lse.data_ptr(), B, Hq, 6, T, d, ctypes.c_float(0.0),
                                         splits, stream)
    assert st == -2, lib.attn_status_string(st)
    st = lib.attn_decode_splitkv_noalloc(q.data_ptr() + 2, kv.data_ptr(), kv.data_ptr(),
                                         o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, T, d,
                                         ctypes.c_float(0.0), splits, stream)
    assert st == -3, lib.attn_status_string(st)


def test_python_binding_of_the_same_name():
    from io_aware_softmax_b200 import attn_decode_splitkv, attn_decode_splitkv_noalloc
    B, Hq, Hkv, T, d = 3, 8, 2, 1000, 128
    q = workloads.randn_bf16((B, Hq, 1, d), 77, 0).cuda()
    kc = workloads.randn_bf16((B, Hkv, T, d), 77, 1).cuda()
    vc = workloads.randn_bf16((B, Hkv, T, d), 77, 2).cuda()
    o, lse = attn_decode_splitkv_noalloc(q, kc, vc, num_splits=6)
    o_ref, lse_ref = attn_decode_splitkv(q, kc, vc, num_splits=6)
    assert device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
