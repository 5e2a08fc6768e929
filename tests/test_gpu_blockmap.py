"""The device tile map (attn_blockmap) equals the oracle's element-by-element map bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from io_aware_softmax_b200 import attn_blockmap, device_status

pytestmark = pytest.mark.gpu


def _check(B, N, mask, window=0, docs=None, Nk=None):
    Nk = N if Nk is None else Nk
    doc_t = None if docs is None else torch.tensor(docs, dtype=torch.int32, device="cuda")
    got = attn_blockmap(B, N, Nk, mask=mask, window=window, doc_offsets=doc_t, device="cuda")
    assert device_status() == 0
    want = oracle.tile_map(B, N, Nk, mask, window, docs)
    assert np.array_equal(got.cpu().numpy(), want)
    return want


@pytest.mark.parametrize("N", [1, 100, 128, 129, 1000, 1025])
@pytest.mark.parametrize("mask", [0, 1])
def test_none_and_causal(N, mask):
    _check(2, N, mask)


def test_non_square_unmasked():
    _check(1, 300, 0, Nk=1000)


@pytest.mark.parametrize("window", [0, 1, 127, 128, 300, 2000])
def test_sliding(window):
    _check(1, 1500, 2, window=window)


@pytest.mark.parametrize("window", [0, 1, 127, 128, 300, 2000])
def test_symmetric_sliding(window):
    _check(2, 1500, 4, window=window)


def test_documents_random():
    for seed in range(4):
        docs = workloads.doc_offsets_for(3000, 1, 700, seed=seed)
        _check(1, 3000, 3, docs=docs)


def test_full_size_workload_maps():
    want = _check(8, 4096, 1)
    assert (want == 2).sum() // 8 == 496 and (want == 1).sum() // 8 == 32
    want = _check(4, 16384, 2, window=1024)
    assert (want == 2).sum() // 4 == 868 and (want == 1).sum() // 4 == 248
    _check(1, 32768, 3, docs=workloads.doc_offsets_for(32768))
