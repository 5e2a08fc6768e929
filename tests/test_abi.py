"""The C-ABI library builds for sm_100a, loads, and exports every symbol include/attn.h
declares.  Only calls that return before any CUDA work run here (no GPU on this host)."""
import ctypes
import os
import re

import pytest

from io_aware_softmax_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def header_symbols():
    text = open(HEADER, encoding="utf-8").read()
    return re.findall(r"ATTN_API\s+[A-Za-z_][\w\s\*]*?\b(attn_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_header_declares_the_entry_points():
    syms = header_symbols()
    for name in ["attn_fwd", "attn_blockmap", "attn_decode_splitkv", "attn_decode_merge",
                 "attn_decode_workspace_bytes", "attn_decode_default_splits",
                 "attn_get_device_status", "attn_status_string"]:
        assert name in syms
    assert set(syms) == set(_lib.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name
    # exported with C linkage, nothing else leaks from the internal namespace
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(header_symbols()) <= exported
    assert not [s for s in exported if s.startswith("_ZN4attn")]


def test_built_for_sm100a_only():
    log = open(os.path.join(os.path.dirname(_lib.LIB_PATH), "ptxas_info.txt")).read()
    assert "for 'sm_100a'" in log
    assert re.search(r"for 'sm_(?!100a)", log) is None
    regs = build.check_register_budget(log)
    for frag, source, big, other in build.SPLIT_KERNELS:
        hits = [r for k, r in regs.items() if frag in k]
        need = build.split_regs(source, big, other)
        assert hits and all(r * build.SPLIT_THREADS >= need for r in hits), frag


def _spills_by_kernel(log):
    out, current = {}, None
    for line in log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and current:
            out[current] = int(m.group(1))
    return out


def test_no_spills_in_the_workload_kernels():
    # d=128 prefill, every decode variant, merge and tile map: no spills; the d=64 prefill
    # variant (not a workload shape) is allowed a few bytes.
    log = open(os.path.join(os.path.dirname(_lib.LIB_PATH), "ptxas_info.txt")).read()
    assert "setmaxnreg' ignored" not in log
    sp = _spills_by_kernel(log)
    assert sp
    for name, b in sp.items():
        if "attn_fwd_sm100_kernelILi64" in name:
            assert b <= 64, (name, b)
        else:
            assert b == 0, (name, b)


def test_status_strings_and_version(lib):
    assert lib.attn_status_string(0) == b"ok"
    assert lib.attn_status_string(-2) == b"unsupported configuration"
    assert lib.attn_status_string(12345) == b"unknown status"
    assert lib.attn_version() >= 100


def test_validation_happens_before_any_launch(lib):
    f = lib.attn_fwd
    P = ctypes.c_void_p(16)       # never dereferenced: every call below fails validation first
    # head dim outside {64, 128}
    assert f(P, P, P, P, P, 1, 2, 2, 8, 8, 96, 0.0, 0, 0, 0.0, None, 0, None) == -2
    # Hq not a multiple of Hkv
    assert f(P, P, P, P, P, 1, 3, 2, 8, 8, 64, 0.0, 0, 0, 0.0, None, 0, None) == -2
    # a mask needs Nq == Nk
    assert f(P, P, P, P, P, 1, 2, 2, 8, 9, 64, 0.0, 1, 0, 0.0, None, 0, None) == -2
    # unknown mask kind, negative window, document mask without offsets
    assert f(P, P, P, P, P, 1, 2, 2, 8, 8, 64, 0.0, 7, 0, 0.0, None, 0, None) == -1
    assert f(P, P, P, P, P, 1, 2, 2, 8, 8, 64, 0.0, 5, 0, 0.0, None, 0, None) == -1
    assert f(P, P, P, P, P, 1, 2, 2, 8, 8, 64, 0.0, 4, -1, 0.0, None, 0, None) == -1
    assert f(P, P, P, P, P, 1, 2, 2, 8, 9, 64, 0.0, 4, 3, 0.0, None, 0, None) == -2
    assert f(P, P, P, P, P, 1, 2, 2, 8, 8, 64, 0.0, 2, -1, 0.0, None, 0, None) == -1
    assert f(P, P, P, P, P, 1, 2, 2, 8, 8, 64, 0.0, 3, 0, 0.0, None, 0, None) == -1
    # negative sizes
    assert f(P, P, P, P, P, -1, 2, 2, 8, 8, 64, 0.0, 0, 0, 0.0, None, 0, None) == -1
    # misaligned pointer
    Q = ctypes.c_void_p(24)
    assert f(Q, P, P, P, P, 1, 2, 2, 8, 8, 64, 0.0, 0, 0, 0.0, None, 0, None) == -3
    # empty problems are a no-op success
    assert f(None, None, None, None, None, 0, 2, 2, 8, 8, 64, 0.0, 0, 0, 0.0, None, 0, None) == 0
    assert f(None, None, None, None, None, 1, 2, 2, 0, 0, 64, 0.0, 1, 0, 0.0, None, 0, None) == 0


def test_decode_validation_and_workspace(lib):
    d = lib.attn_decode_splitkv
    P = ctypes.c_void_p(16)
    assert d(P, P, P, P, P, 1, 64, 2, 8, 128, 0.0, 1, P, 1 << 20, None) == -2      # G = 32
    assert d(P, P, P, P, P, 1, 4, 2, 8, 80, 0.0, 1, P, 1 << 20, None) == -2        # d = 80
    assert d(P, P, P, P, P, 1, 4, 2, 8, 128, 0.0, 2, None, 0, None) == -6          # no workspace
    assert d(P, P, P, P, P, 1, 4, 2, 8, 128, 0.0, 2, P, 10, None) == -6            # too small
    need = lib.attn_decode_workspace_bytes(64, 32, 128, 15)
    rows = 64 * 32 * 15
    assert need == ((rows * 128 * 4 + 255) // 256) * 256 + rows * 4
    assert lib.attn_decode_workspace_bytes(0, 32, 128, 15) == 0
    m = lib.attn_decode_merge
    assert m(P, P, P, P, 4, 3, 96, None) == -2
    assert m(P, P, P, P, 4, 0, 128, None) == -1
    assert m(None, None, None, None, 0, 3, 128, None) == 0


def test_blockmap_validation(lib):
    b = lib.attn_blockmap
    assert b(1, 8, 9, 1, 0, None, 0, ctypes.c_void_p(16), None) == -2
    assert b(1, 8, 8, 3, 0, None, 0, ctypes.c_void_p(16), None) == -1
    assert b(1, 8, 8, 4, -2, None, 0, ctypes.c_void_p(16), None) == -1
    assert b(0, 8, 8, 1, 0, None, 0, None, None) == 0


def test_default_split_heuristic(lib):
    # 512 KV heads on 148 SMs x 2 resident CTAs: 15 splits fill 26 waves to 99.8 %
    s = lib.attn_decode_default_splits(64, 8, 32768, 0)
    items = 64 * 8 * s
    slots = 148 * 2
    waves = -(-items // slots)
    assert items / (waves * slots) >= 0.99 and 32768 // s >= 128
    assert lib.attn_decode_default_splits(1, 1, 100, 0) == 1
    assert lib.attn_decode_default_splits(1, 1, 0, 0) == 1


def test_alibi_entry_validation(lib):
    a = lib.attn_fwd_alibi
    P = ctypes.c_void_p(16)
    # slopes must be 4-byte aligned; a bias with a soft-cap is not supported
    assert a(P, P, P, P, P, 1, 2, 2, 8, 8, 64, 0.0, 1, 0, 0.0, None, 0, ctypes.c_void_p(18),
             None) == -3
    assert a(P, P, P, P, P, 1, 2, 2, 8, 8, 64, 0.0, 1, 0, 30.0, None, 0, P, None) == -2
    # the shared checks still come first, and empty problems are a no-op
    assert a(P, P, P, P, P, 1, 2, 2, 8, 8, 96, 0.0, 1, 0, 0.0, None, 0, P, None) == -2
    assert a(None, None, None, None, None, 0, 2, 2, 8, 8, 64, 0.0, 1, 0, 0.0, None, 0, P,
             None) == 0


def test_paged_decode_validation(lib):
    f = lib.attn_decode_paged
    P = ctypes.c_void_p(16)
    I4 = ctypes.c_void_p(20)          # 4-byte aligned, not 16
    # (q, k_pages, v_pages, table, lens, o, lse, B, Hq, Hkv, pages, page_size, max_pages, d,
    #  scale, splits, ws, ws_bytes, stream)
    assert f(P, P, P, I4, I4, P, P, 2, 8, 2, 10, 48, 4, 128, 0.0, 1, P, 1 << 20, None) == -2
    assert f(P, P, P, I4, I4, P, P, 2, 8, 2, 10, 64, 4, 96, 0.0, 1, P, 1 << 20, None) == -2
    assert f(P, P, P, I4, I4, P, P, 2, 8, 2, 10, 0, 4, 128, 0.0, 1, P, 1 << 20, None) == -1
    assert f(P, P, P, I4, None, P, P, 2, 8, 2, 10, 64, 4, 128, 0.0, 1, P, 1 << 20, None) == -1
    assert f(P, P, P, I4, ctypes.c_void_p(22), P, P, 2, 8, 2, 10, 64, 4, 128, 0.0, 1, P,
             1 << 20, None) == -3
    assert f(P, P, P, I4, I4, P, P, 2, 64, 2, 10, 64, 4, 128, 0.0, 1, P, 1 << 20, None) == -2
    assert f(P, P, P, I4, I4, P, P, 2, 8, 2, 10, 64, 4, 128, 0.0, 2, None, 0, None) == -6
    assert f(None, None, None, None, None, None, None, 0, 8, 2, 10, 64, 4, 128, 0.0, 1, None, 0,
             None) == 0


def test_backward_validation(lib):
    f = lib.attn_bwd
    P = ctypes.c_void_p(16)
    args = lambda **kw: [kw.get("q", P), P, P, P, P, P, P, P, P, 1, 2, 2, 64, 64,
                         kw.get("d", 128), 0.0, kw.get("mask", 1), 0, kw.get("cap", 0.0), None, 0,
                         kw.get("ws", P), kw.get("wsb", 1 << 20), None]
    assert f(*args(d=96)) == -2
    assert f(*args(cap=float("nan"))) == -1
    assert f(*args(mask=9)) == -1
    assert f(*args(q=ctypes.c_void_p(24))) == -3
    assert f(*args(ws=None, wsb=0)) == -6
    assert f(*args(wsb=10)) == -6
    assert lib.attn_bwd_workspace_bytes(2, 4, 100) == 2 * ((2 * 4 * 100 * 4 + 255) // 256 * 256)
    assert lib.attn_bwd_workspace_bytes(0, 4, 100) == 0


def test_backward_alibi_validation(lib):
    # the same checks as attn_bwd, plus 4-byte alignment of the slopes; no launch happens
    f = lib.attn_bwd_alibi
    P = ctypes.c_void_p(16)
    args = lambda **kw: [P, P, P, P, P, P, P, P, P, 1, 2, 2, 64, 64, kw.get("d", 128), 0.0, 1, 0,
                         kw.get("cap", 0.0), None, 0, kw.get("slopes", P), P, 1 << 20, None]
    assert f(*args(slopes=ctypes.c_void_p(18))) == -3
    assert f(*args(d=96)) == -2
    assert f(*args(cap=30.0)) == -2


def test_fp8_entry_validation(lib):
    f = lib.attn_fwd_fp8
    P = ctypes.c_void_p(16)
    # (q8, k8, vt8, qs, ks, vs, o, lse, B, Hq, Hkv, Nq, Nk, nk_pad, d, scale, mask, window,
    #  docs, num_docs, stream)
    assert f(P, P, P, P, P, P, P, P, 1, 2, 2, 64, 64, 64, 64, 0.0, 1, 0, None, 0, None) == -2
    assert f(P, P, P, P, P, P, P, P, 1, 2, 2, 64, 64, 60, 128, 0.0, 1, 0, None, 0, None) == -1
    assert f(P, P, P, P, P, P, P, P, 1, 2, 2, 64, 64, 72, 128, 0.0, 1, 0, None, 0, None) == -1
    assert f(P, P, P, P, P, P, P, P, 1, 3, 2, 64, 64, 64, 128, 0.0, 1, 0, None, 0, None) == -2
    assert f(None, None, None, None, None, None, None, None, 0, 2, 2, 64, 64, 64, 128, 0.0, 1, 0,
             None, 0, None) == 0
    q = lib.attn_quantize_fp8
    assert q(P, P, P, 1, 1, 8, 96, 128, 0, 0, None, None) == -2
    assert q(P, P, P, 1, 1, 8, 128, 0, 0, 0, None, None) == -1
    assert q(P, P, P, 1, 1, 8, 128, 128, 1, 4, None, None) == -1      # n_pad < N
    assert q(ctypes.c_void_p(24), P, P, 1, 1, 8, 128, 128, 0, 0, None, None) == -3
