"""Parity of split-KV decode and the merge kernel (through the C ABI) with the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from io_aware_softmax_b200 import (attn_decode, attn_merge, decode_workspace_bytes,
                                   default_splits, device_status)
from tests.gpu_common import compare, f64

pytestmark = pytest.mark.gpu


def _decode_case(B, Hq, Hkv, T, d, splits, seed, std=1.0):
    q = workloads.randn_bf16((B, Hq, 1, d), seed, 0, std).cuda()
    kc = workloads.randn_bf16((B, Hkv, T, d), seed, 1, std).cuda()
    vc = workloads.randn_bf16((B, Hkv, T, d), seed, 2).cuda()     # std widens q and K only
    o, lse = attn_decode(q, kc, vc, num_splits=splits)
    assert device_status() == 0
    O_ref, L_ref = oracle.attention(f64(q), f64(kc), f64(vc))
    return compare(o, lse, O_ref, L_ref, f"decode B{B} Hq{Hq} Hkv{Hkv} T{T} d{d} S{splits}")


@pytest.mark.parametrize("T", [1, 7, 64, 65, 1000, 4097])
@pytest.mark.parametrize("splits", [1, 3, 8])
def test_lengths_and_splits(T, splits):
    _decode_case(2, 8, 2, T, 128, splits, seed=T * 7 + splits)


@pytest.mark.parametrize("G", [1, 2, 4, 8, 12, 16])
def test_group_sizes(G):
    _decode_case(2, 2 * G, 2, 1500, 128, 5, seed=G)


@pytest.mark.parametrize("d", [64, 128])
def test_head_dims_and_default_splits(d):
    _decode_case(3, 8, 2, 3000, d, None, seed=d)


def test_more_splits_than_tokens_and_large_scores():
    _decode_case(1, 4, 1, 40, 128, 64, seed=5, std=3.0)


def test_workspace_holds_split_partials_that_merge_to_the_output():
    B, Hq, Hkv, T, d, S = 2, 8, 2, 2000, 128, 6
    q = workloads.randn_bf16((B, Hq, 1, d), 77, 0).cuda()
    kc = workloads.randn_bf16((B, Hkv, T, d), 77, 1).cuda()
    vc = workloads.randn_bf16((B, Hkv, T, d), 77, 2).cuda()
    ws = torch.empty(decode_workspace_bytes(B, Hq, d, S), dtype=torch.uint8, device="cuda")
    o, lse = attn_decode(q, kc, vc, num_splits=S, workspace=ws)
    assert device_status() == 0
    rows = B * Hq * S
    o_bytes = ((rows * d * 4 + 255) // 256) * 256
    o_part = ws[:rows * d * 4].view(torch.float32).view(B, Hq, S, d)
    lse_part = ws[o_bytes:o_bytes + rows * 4].view(torch.float32).view(B, Hq, S)
    # the partials are the oracle's per-split results; the kernel cuts at 64-row tiles
    _, _, O_parts, L_parts = oracle.decode_splitkv(f64(q), f64(kc), f64(vc), S, tile=64)
    compare(o_part, lse_part, O_parts[:, :, 0], L_parts[:, :, 0], "split partials")


def test_merge_kernel_against_oracle_rule():
    rng = np.random.default_rng(3)
    rows, S, d = 37, 9, 128
    o_part = rng.standard_normal((rows, S, d))
    lse_part = rng.standard_normal((rows, S)) * 4
    lse_part[rng.random((rows, S)) < 0.3] = -np.inf        # empty splits carry weight 0
    lse_part[5, :] = -np.inf                                # a row with no key at all
    o_t = torch.tensor(o_part, dtype=torch.float32, device="cuda")
    l_t = torch.tensor(lse_part, dtype=torch.float32, device="cuda")
    o, lse = attn_merge(o_t, l_t)
    assert device_status() == 0
    O_ref, L_ref = oracle.merge_partials(f64(o_t), f64(l_t))
    compare(o, lse, O_ref, L_ref, "merge")


def test_decode_workload_full_size_sampled():
    w = workloads.DECODE
    q, kc, vc = workloads.make_inputs(w, device="cuda")
    S = default_splits(w.B, w.Hkv, w.Nk, torch.cuda.current_device())
    o, lse = attn_decode(q, kc, vc, scale=w.scale, num_splits=S)
    assert device_status() == 0
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(0)
    G = w.Hq // w.Hkv
    picks = {(0, 0), (w.B - 1, w.Hq - 1)} | {(int(rng.integers(w.B)), int(rng.integers(w.Hq)))
                                            for _ in range(4)}
    for b, h in sorted(picks):
        O_ref, L_ref = oracle.attention_head(f64(q[b, h]), np.arange(1), f64(kc[b, h // G]),
                                             f64(vc[b, h // G]), w.scale)
        compare(o[b, h], lse[b, h], O_ref, L_ref, f"decode b{b} h{h}")


def test_empty_cache_gives_zero_and_minus_inf():
    q = workloads.randn_bf16((1, 4, 1, 128), 1, 0).cuda()
    kc = torch.empty((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    o, lse = attn_decode(q, kc, kc, num_splits=1)
    assert device_status() == 0
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
