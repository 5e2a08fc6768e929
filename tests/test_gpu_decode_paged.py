"""Parity of decode over paged, variable-length caches (attn_decode_paged through the C ABI)
with the fp64 oracle's paged decode."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from io_aware_softmax_b200 import attn_decode, attn_decode_paged, device_status
from tests.gpu_common import compare, f64

pytestmark = pytest.mark.gpu


def _paged_inputs(B, Hq, Hkv, page, max_pages, d, lens, seed, spare_pages=3, std=1.0):
    num_pages = B * max_pages + spare_pages
    q = workloads.randn_bf16((B, Hq, 1, d), seed, 0, std, device="cuda")
    kp = workloads.randn_bf16((num_pages, Hkv, page, d), seed, 1, std, device="cuda")
    vp = workloads.randn_bf16((num_pages, Hkv, page, d), seed, 2, device="cuda")  # std: q, K only
    rng = np.random.default_rng(seed)
    table = rng.permutation(num_pages)[: B * max_pages].reshape(B, max_pages).astype(np.int32)
    return (q, kp, vp, torch.from_numpy(table).cuda(),
            torch.tensor(lens, dtype=torch.int32, device="cuda"), table)


def _paged_case(B, Hq, Hkv, page, max_pages, d, lens, splits, seed, std=1.0):
    q, kp, vp, table_t, lens_t, table = _paged_inputs(B, Hq, Hkv, page, max_pages, d, lens, seed,
                                                      std=std)
    o, lse = attn_decode_paged(q, kp, vp, table_t, lens_t, num_splits=splits)
    assert device_status() == 0
    O_ref, L_ref = oracle.decode_paged(f64(q), f64(kp), f64(vp), table, np.asarray(lens))
    return compare(o, lse, O_ref, L_ref,
                   f"paged B{B} Hq{Hq} Hkv{Hkv} page{page} lens{lens} d{d} S{splits}")


@pytest.mark.parametrize("page", [64, 128, 256])
@pytest.mark.parametrize("splits", [1, 3, 7, None])
def test_lengths_pages_and_splits(page, splits):
    max_pages = 2048 // page
    lens = [0, 1, 63, 64, 65, 700, 2047, 2048]
    _paged_case(len(lens), 8, 2, page, max_pages, 128, lens, splits, seed=page + (splits or 0))


@pytest.mark.parametrize("G", [1, 4, 8, 12, 16])
def test_group_sizes(G):
    _paged_case(3, 2 * G, 2, 128, 10, 128, [1000, 1280, 77], 5, seed=G)


@pytest.mark.parametrize("d", [64, 128])
def test_head_dims_and_large_scores(d):
    _paged_case(2, 8, 2, 64, 20, d, [1279, 300], None, seed=d, std=3.0)


def test_lengths_past_the_table_are_clamped_and_negative_lengths_are_empty():
    # seq_lens above max_pages * page_size read only the table's pages; negative means empty
    B, Hq, Hkv, page, max_pages, d = 3, 4, 1, 64, 4, 128
    q, kp, vp, table_t, _, table = _paged_inputs(B, Hq, Hkv, page, max_pages, d, [0, 0, 0], 9)
    lens = torch.tensor([10_000, -5, 100], dtype=torch.int32, device="cuda")
    o, lse = attn_decode_paged(q, kp, vp, table_t, lens, num_splits=3)
    assert device_status() == 0
    O_ref, L_ref = oracle.decode_paged(f64(q), f64(kp), f64(vp), table,
                                       np.array([page * max_pages, 0, 100]))
    compare(o, lse, O_ref, L_ref, "clamped lengths")


def test_one_page_per_sequence_is_the_contiguous_cache():
    # the contiguous layout [B, Hkv, T, d] is the paged layout with one page per sequence
    B, Hq, Hkv, T, d = 4, 16, 4, 1024, 128
    q = workloads.randn_bf16((B, Hq, 1, d), 31, 0).cuda()
    kc = workloads.randn_bf16((B, Hkv, T, d), 31, 1).cuda()
    vc = workloads.randn_bf16((B, Hkv, T, d), 31, 2).cuda()
    table = torch.arange(B, dtype=torch.int32, device="cuda").view(B, 1)
    lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    o1, l1 = attn_decode_paged(q, kc, vc, table, lens, num_splits=4)
    o2, l2 = attn_decode(q, kc, vc, num_splits=4)
    assert device_status() == 0
    O_ref, L_ref = oracle.attention(f64(q), f64(kc), f64(vc))
    compare(o1, l1, O_ref, L_ref, "one page per sequence")
    compare(o2, l2, O_ref, L_ref, "contiguous")


def test_unsupported_page_size_raises():
    q, kp, vp, table_t, lens_t, _ = _paged_inputs(1, 4, 1, 64, 2, 128, [100], 3)
    with pytest.raises(Exception) as e:
        attn_decode_paged(q, kp[:, :, :48].contiguous(), vp[:, :, :48].contiguous(), table_t,
                          lens_t)
    assert "unsupported" in str(e.value).lower()


def test_full_size_paged_cache_sampled():
    # the decode workload's sizes (B=64, Hq=32, Hkv=8, d=128) on a paged cache of 256-row
    # pages in random placement, with per-sequence lengths up to 32768
    B, Hq, Hkv, page, max_pages, d = 64, 32, 8, 256, 128, 128
    rng = np.random.default_rng(17)
    lens = rng.integers(1, page * max_pages + 1, size=B).astype(np.int32)
    lens[0], lens[1] = page * max_pages, 1
    q, kp, vp, table_t, lens_t, table = _paged_inputs(B, Hq, Hkv, page, max_pages, d, lens, 41,
                                                      spare_pages=0)
    o, lse = attn_decode_paged(q, kp, vp, table_t, lens_t)
    assert device_status() == 0
    for b in (0, 1, 33, 63):
        T = int(lens[b])
        n = -(-T // page)
        # only this sequence's pages go to the host; the oracle gathers them in table order
        K = oracle.gather_paged(f64(kp[table_t[b, :n].long()]), np.arange(n), T)
        V = oracle.gather_paged(f64(vp[table_t[b, :n].long()]), np.arange(n), T)
        for h in (0, 5, 31):
            O_ref, L_ref = oracle.attention_head(f64(q[b, h]), np.arange(1), K[h // 4], V[h // 4],
                                                 oracle.default_scale(d))
            compare(o[b, h], lse[b, h], O_ref, L_ref, f"full paged b{b} h{h}")
