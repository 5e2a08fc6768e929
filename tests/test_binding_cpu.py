"""The Python binding's argument checks, run on the CPU against a recording stand-in for the
library: valid calls reach the library once with the sizes the C entry points take, and
tensors whose shape, dtype or device disagree with the inputs are refused before any call
(the library reads and writes the extents its size arguments imply, so a mismatched tensor
would otherwise be overrun on the device)."""
import contextlib

import pytest
import torch

from io_aware_softmax_b200 import api

BF16, F32, U8, I32, E4M3 = torch.bfloat16, torch.float32, torch.uint8, torch.int32, torch.float8_e4m3fn


class FakeLib:
    """Records each entry point's arguments; every call succeeds."""

    def __init__(self):
        self.calls = []

    def attn_bwd_workspace_bytes(self, B, Hq, Nq):
        return 2 * ((B * Hq * Nq * 4 + 255) // 256 * 256)

    def attn_decode_workspace_bytes(self, B, Hq, d, S):
        return B * Hq * S * (d + 1) * 4

    def attn_decode_default_splits(self, B, Hkv, T, dev):
        return 4

    def attn_status_string(self, st):
        return b"stand-in"

    def __getattr__(self, name):
        if not name.startswith("attn_"):
            raise AttributeError(name)

        def record(*args):
            self.calls.append((name, args))
            return 0
        return record


@pytest.fixture
def lib(monkeypatch):
    fake = FakeLib()
    monkeypatch.setattr(api._lib, "load", lambda *a, **k: fake)
    monkeypatch.setattr(api, "_on_gpu", lambda t, name: None)
    monkeypatch.setattr(api, "_device", lambda t: contextlib.nullcontext())
    monkeypatch.setattr(api, "_stream", lambda device, stream=None: 0)
    monkeypatch.setattr(api, "_index", lambda t: 0)
    return fake


def z(shape, dtype=BF16, device="cpu"):
    return torch.zeros(shape, dtype=dtype, device=device)


def only_call(fake, name):
    assert [c[0] for c in fake.calls] == [name], fake.calls
    return fake.calls[0][1]


# ------------------------------------------------------------------ valid calls go through

def test_fwd_sizes_and_preallocated_views(lib):
    B, Hq, Hkv, N, d = 2, 6, 3, 300, 128
    o_buf = z(B * Hq * N * d + 64)
    l_buf = z(B * Hq * N + 16, F32)
    o, lse = api.attn_fwd(z((B, Hq, N, d)), z((B, Hkv, N, d)), z((B, Hkv, N, d)), mask="causal",
                          out=o_buf[: B * Hq * N * d].view(B, Hq, N, d),
                          lse=l_buf[: B * Hq * N].view(B, Hq, N))
    args = only_call(lib, "attn_fwd")
    assert args[5:11] == (B, Hq, Hkv, N, N, d)
    assert args[12] == 1


def test_fwd_alibi_and_documents(lib):
    docs = torch.tensor([0, 100, 300], dtype=I32)
    api.attn_fwd(z((1, 4, 300, 64)), z((1, 2, 300, 64)), z((1, 2, 300, 64)),
                 mask="document_causal", doc_offsets=docs, alibi_slopes=z((4,), F32))
    args = only_call(lib, "attn_fwd_alibi")
    assert args[16] == 2                                     # num_docs


def test_bwd_with_every_buffer_supplied(lib):
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 128
    q, k = z((B, Hq, N, d)), z((B, Hkv, N, d))
    ws = z(api.bwd_workspace_bytes(B, Hq, N), U8)
    api.attn_bwd(q, k, z(k.shape), z(q.shape), z((B, Hq, N), F32), z(q.shape), mask="causal",
                 dq=z(q.shape), dk=z(k.shape), dv=z(k.shape), workspace=ws)
    args = only_call(lib, "attn_bwd")
    assert args[9:15] == (B, Hq, Hkv, N, N, d)
    assert args[22] == ws.numel()


def test_fp8_forward_from_quantizer_shapes(lib):
    B, Hq, Hkv, N, d = 1, 4, 2, 500, 128
    q8, qs = api.quantize_fp8(z((B, Hq, N, d)), block_rows=128, signs=z((d,), F32))
    k8, ks = api.quantize_fp8(z((B, Hkv, N, d)), block_rows=128)
    vt8, vs = api.quantize_fp8(z((B, Hkv, N, d)), block_rows=N, transpose=True)
    assert tuple(vt8.shape) == (B, Hkv, d, 512) and tuple(vs.shape) == (B, Hkv, 1)
    api.attn_fwd_fp8(q8, qs, k8, ks, vt8, vs[:, :, 0], mask="causal")
    names = [c[0] for c in lib.calls]
    assert names == ["attn_quantize_fp8"] * 3 + ["attn_fwd_fp8"]
    assert lib.calls[3][1][8:15] == (B, Hq, Hkv, N, N, 512, d)


def test_decode_paged_and_merge(lib):
    B, Hq, Hkv, T, d, S = 2, 8, 2, 700, 128, 3
    ws = z(api.decode_workspace_bytes(B, Hq, d, S), U8)
    api.attn_decode(z((B, Hq, 1, d)), z((B, Hkv, T, d)), z((B, Hkv, T, d)), num_splits=S,
                    workspace=ws, out=z((B, Hq, 1, d)), lse=z((B, Hq, 1), F32))
    api.attn_decode_paged(z((B, Hq, 1, d)), z((12, Hkv, 64, d)), z((12, Hkv, 64, d)),
                          z((B, 6), I32), z((B,), I32), num_splits=S, workspace=ws,
                          out=z((B, Hq, 1, d)), lse=z((B, Hq, 1), F32))
    api.attn_merge(z((37, 9, d), F32), z((37, 9), F32))
    api.attn_blockmap(2, 300, 300, mask="causal", device="cpu")
    assert [c[0] for c in lib.calls] == ["attn_decode_splitkv", "attn_decode_paged",
                                         "attn_decode_merge", "attn_blockmap"]
    assert lib.calls[0][1][5:11] == (B, Hq, Hkv, T, d, 0.0)


# ------------------------------------------------------------------ mismatches are refused

@pytest.mark.parametrize("case", [
    "v_rows", "k_batch", "k_dim", "out_shape", "out_dtype", "lse_shape", "lse_strided"])
def test_fwd_mismatch_is_refused(lib, case):
    q, k, v = z((1, 4, 128, 64)), z((1, 2, 128, 64)), z((1, 2, 128, 64))
    kw = {}
    if case == "v_rows":
        v = z((1, 2, 100, 64))
    elif case == "k_batch":
        k, v = z((2, 2, 128, 64)), z((2, 2, 128, 64))
    elif case == "k_dim":
        k, v = z((1, 2, 128, 128)), z((1, 2, 128, 128))
    elif case == "out_shape":
        kw["out"] = z((1, 4, 127, 64))
    elif case == "out_dtype":
        kw["out"] = z((1, 4, 128, 64), F32)
    elif case == "lse_shape":
        kw["lse"] = z((1, 4, 64), F32)
    elif case == "lse_strided":
        kw["lse"] = z((1, 4, 256), F32)[:, :, ::2]
    with pytest.raises((ValueError, TypeError)):
        api.attn_fwd(q, k, v, **kw)
    assert lib.calls == []


@pytest.mark.parametrize("which", ["dq", "dk", "dv"])
def test_bwd_gradient_buffer_of_the_wrong_shape_is_refused(lib, which):
    q, k = z((1, 4, 200, 64)), z((1, 2, 200, 64))
    kw = {which: z((1, 4, 199, 64))}
    with pytest.raises(ValueError):
        api.attn_bwd(q, k, z(k.shape), z(q.shape), z((1, 4, 200), F32), z(q.shape), **kw)
    assert lib.calls == []


def test_bwd_strided_workspace_is_refused(lib):
    q, k = z((1, 4, 200, 64)), z((1, 2, 200, 64))
    ws = z(2 * api.bwd_workspace_bytes(1, 4, 200), U8)[::2]
    with pytest.raises(ValueError):
        api.attn_bwd(q, k, z(k.shape), z(q.shape), z((1, 4, 200), F32), z(q.shape), workspace=ws)
    assert lib.calls == []


@pytest.mark.parametrize("case", ["q_scales", "k_scales", "v_scales", "vt8", "k8"])
def test_fp8_mismatch_is_refused(lib, case):
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 128
    a = {"q8": z((B, Hq, N, d), E4M3), "qs": z((B, Hq, 3), F32), "k8": z((B, Hkv, N, d), E4M3),
         "ks": z((B, Hkv, 3), F32), "vt8": z((B, Hkv, d, 304), E4M3), "vs": z((B, Hkv), F32)}
    if case == "q_scales":
        a["qs"] = z((B, Hq, 2), F32)
    elif case == "k_scales":
        a["ks"] = z((B, Hq, 3), F32)
    elif case == "v_scales":
        a["vs"] = z((B, Hq), F32)
    elif case == "vt8":
        a["vt8"] = z((B, Hkv, 64, 304), E4M3)
    elif case == "k8":
        a["k8"] = z((B, Hkv, N, 64), E4M3)
    with pytest.raises(ValueError):
        api.attn_fwd_fp8(a["q8"], a["qs"], a["k8"], a["ks"], a["vt8"], a["vs"])
    assert lib.calls == []


def test_quantizer_sign_count_and_block_rows(lib):
    with pytest.raises(ValueError):
        api.quantize_fp8(z((1, 2, 64, 128)), signs=z((64,), F32))
    with pytest.raises(ValueError):
        api.quantize_fp8(z((1, 2, 64, 128)), block_rows=0)
    assert lib.calls == []


def test_decode_mismatches_are_refused(lib):
    q = z((2, 8, 1, 128))
    with pytest.raises(ValueError):
        api.attn_decode(q, z((2, 2, 700, 128)), z((2, 2, 699, 128)))
    with pytest.raises(ValueError):
        api.attn_decode(q, z((1, 2, 700, 128)), z((1, 2, 700, 128)))
    with pytest.raises(ValueError):
        api.attn_decode(q, z((2, 2, 700, 128)), z((2, 2, 700, 128)), lse=z((2, 8), F32))
    with pytest.raises(ValueError):
        api.attn_decode_paged(q, z((12, 2, 64, 128)), z((12, 2, 64, 64)), z((2, 6), I32),
                              z((2,), I32))
    with pytest.raises(ValueError):
        api.attn_merge(z((37, 9, 128), F32), z((37, 8), F32))
    with pytest.raises(ValueError):
        api.attn_blockmap(2, 300, 300, device="cpu", out=z((2, 3, 2), U8))
    assert lib.calls == []


def test_tensors_on_another_device_are_refused(lib):
    # the meta device stands in for a second GPU: only the device differs
    q = z((1, 4, 128, 64))
    k_meta = z((1, 2, 128, 64), device="meta")
    with pytest.raises(ValueError, match="meta"):
        api.attn_fwd(q, k_meta, z((1, 2, 128, 64)))
    with pytest.raises(ValueError, match="meta"):
        api.attn_fwd(q, z((1, 2, 128, 64)), z((1, 2, 128, 64)),
                     out=z((1, 4, 128, 64), device="meta"))
    assert lib.calls == []


# ------------------------------------------------------------------ one binding per entry point

def test_every_declared_entry_point_has_a_binding_of_the_same_name():
    import re
    from pathlib import Path

    import io_aware_softmax_b200 as pkg
    header = (Path(__file__).resolve().parents[1] / "include" / "attn.h").read_text()
    names = re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", header)
    assert len(names) >= 16, names
    missing = [n for n in names if not callable(getattr(pkg, n, None))]
    assert not missing, missing
    assert set(names) <= set(pkg.__all__)


def test_noalloc_and_alibi_bindings(lib):
    q, kc = z((2, 8, 1, 128)), z((2, 2, 700, 128))
    api.attn_decode_splitkv_noalloc(q, kc, z(kc.shape), num_splits=5)
    api.attn_fwd_alibi(z((1, 4, 64, 64)), z((1, 2, 64, 64)), z((1, 2, 64, 64)), z((4,), F32),
                       mask="causal")
    assert [c[0] for c in lib.calls] == ["attn_decode_splitkv_noalloc", "attn_fwd_alibi"]
    assert lib.calls[0][1][5:12] == (2, 8, 2, 700, 128, 0.0, 5)
    with pytest.raises(ValueError):
        api.attn_decode_splitkv_noalloc(q, kc, z((2, 2, 600, 128)))
    with pytest.raises(ValueError):
        api.attn_decode_splitkv_noalloc(q, kc, z(kc.shape), lse=z((2, 8), F32))
    assert len(lib.calls) == 2
