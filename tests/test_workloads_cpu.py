"""The seeded input generators that the oracle and the CUDA path share (no attention
arithmetic lives there), checked on the CPU: reproducible bits, independent streams, the
"N(0,1)*2" reading (an exact doubling before the bf16 rounding), and the five workloads'
sizes."""
import numpy as np
import pytest
import torch

import workloads


def test_draws_are_reproducible_bit_for_bit():
    a = workloads.randn_bf16((2, 3, 17, 8), 5, 1)
    b = workloads.randn_bf16((2, 3, 17, 8), 5, 1)
    assert a.dtype == torch.bfloat16 and torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_each_leading_slice_has_its_own_stream():
    # slice b does not depend on how many slices are drawn, so a full-size tensor and a
    # smaller batch share their first slices
    big = workloads.randn_bf16((4, 2, 33, 16), 7, 2)
    small = workloads.randn_bf16((2, 2, 33, 16), 7, 2)
    assert torch.equal(big[:2], small)
    assert not torch.equal(big[0], big[1])


@pytest.mark.parametrize("other", [(8, 1), (7, 3)])
def test_seeds_and_tensor_ids_give_different_draws(other):
    a = workloads.randn_bf16((1, 2, 64, 16), 7, 1)
    b = workloads.randn_bf16((1, 2, 64, 16), *other)
    assert not torch.equal(a, b)


def test_scaled_draws_are_the_doubled_unit_draws():
    # doubling is exact in fp32 and commutes with rounding to bf16
    one = workloads.randn_bf16((2, 2, 50, 16), 3, 0)
    two = workloads.randn_bf16((2, 2, 50, 16), 3, 0, std=2.0)
    assert torch.equal((one.float() * 2).bfloat16(), two)


def test_moments_of_a_large_draw():
    x = workloads.randn_bf16((1, 8, 4096, 64), 11, 0).float().numpy()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    # bf16 rounding: every value is representable with 8 significant bits
    bits = torch.from_numpy(x).view(torch.int32).numpy()
    assert np.all(bits & 0xFFFF == 0)


@pytest.mark.parametrize("w,shape", [
    (workloads.TINY, (1, 2, 2, 128, 128, 64)),
    (workloads.CAUSAL_MHA, (8, 32, 32, 4096, 4096, 128)),
    (workloads.SWA_GQA, (4, 32, 8, 16384, 16384, 128)),
    (workloads.DOC_SOFTCAP, (1, 16, 16, 32768, 32768, 128)),
    (workloads.DECODE, (64, 32, 8, 1, 32768, 128)),
])
def test_workload_sizes(w, shape):
    assert (w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d) == shape
    assert w.scale == pytest.approx(1.0 / np.sqrt(w.d))


def test_workload_hooks():
    assert workloads.SWA_GQA.window == 1024
    assert workloads.DOC_SOFTCAP.softcap == 50.0 and workloads.DOC_SOFTCAP.input_std == 2.0
    docs = workloads.workload_doc_offsets(workloads.DOC_SOFTCAP)
    assert docs[0] == 0 and docs[-1] == 32768 and np.all(np.diff(docs) > 0)


def test_make_inputs_shapes_and_streams():
    q, k, v = workloads.make_inputs(workloads.TINY)
    assert q.shape == (1, 2, 128, 64) and k.shape == v.shape == (1, 2, 128, 64)
    assert not torch.equal(q, k) and not torch.equal(k, v)
