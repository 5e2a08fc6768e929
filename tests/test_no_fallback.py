"""The product path has no CPU or library fallback: without the CUDA library, or given host
tensors, every entry point raises instead of computing anything (runs on the CPU)."""
import pytest
import torch

import io_aware_softmax_b200 as attn
from io_aware_softmax_b200 import _lib


def test_missing_library_raises(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)      # forget a library loaded by other tests
    with pytest.raises(_lib.LibraryMissing):
        _lib.load(str(tmp_path / "libattn_b200.so"))


def test_unloadable_library_raises(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    bad = tmp_path / "libattn_b200.so"
    bad.write_bytes(b"not a shared object")
    with pytest.raises(_lib.LibraryMissing):
        _lib.load(str(bad))


@pytest.mark.parametrize("call", [
    lambda t: attn.attn_fwd(t, t, t),
    lambda t: attn.attn_decode(t[:, :, :1], t, t),
    lambda t: attn.quantize_fp8(t),
    lambda t: attn.attn_bwd(t, t, t, t, torch.zeros(t.shape[:3]), t),
])
def test_host_tensors_are_rejected(call):
    # bf16 host tensors of a valid shape: the binding refuses them before any call into the
    # library, so nothing can silently run on the CPU
    t = torch.zeros((1, 2, 16, 64), dtype=torch.bfloat16)
    with pytest.raises((ValueError, TypeError, _lib.LibraryMissing)):
        call(t)
