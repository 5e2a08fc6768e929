"""Parity of the fused prefill kernel (attn_fwd through the C ABI) with the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from io_aware_softmax_b200 import attn_fwd, device_status
from tests.gpu_common import BF16_UNIT_ROUNDOFF, compare, f64, sample_rows

pytestmark = pytest.mark.gpu

MASK_ID = {"none": 0, "causal": 1, "sliding_causal": 2, "document_causal": 3, "sliding": 4}


def _inputs(B, Hq, Hkv, Nq, Nk, d, seed, std=1.0, v_std=1.0):
    # std widens Q and K (larger scores); V keeps its own spread
    q = workloads.randn_bf16((B, Hq, Nq, d), seed, 0, std).cuda()
    k = workloads.randn_bf16((B, Hkv, Nk, d), seed, 1, std).cuda()
    v = workloads.randn_bf16((B, Hkv, Nk, d), seed, 2, v_std).cuda()
    return q, k, v


def _run_full(B, Hq, Hkv, Nq, Nk, d, mask="none", window=0, softcap=0.0, docs=None, seed=0,
              std=1.0, scale=None, slopes=None, v_std=1.0):
    q, k, v = _inputs(B, Hq, Hkv, Nq, Nk, d, seed, std, v_std)
    doc_t = None if docs is None else torch.tensor(docs, dtype=torch.int32, device="cuda")
    # guard bands around the outputs catch writes past the last row
    o_buf = torch.full((B * Hq * Nq * d + 4096,), float("nan"), dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((B * Hq * Nq + 1024,), float("nan"), dtype=torch.float32, device="cuda")
    o = o_buf[: B * Hq * Nq * d].view(B, Hq, Nq, d)
    lse = l_buf[: B * Hq * Nq].view(B, Hq, Nq)
    slopes_t = None if slopes is None else torch.tensor(slopes, dtype=torch.float32, device="cuda")
    attn_fwd(q, k, v, scale=scale, mask=mask, window=window, softcap=softcap, doc_offsets=doc_t,
             alibi_slopes=slopes_t, out=o, lse=lse)
    assert device_status() == 0
    assert torch.isnan(o_buf[B * Hq * Nq * d:]).all() and torch.isnan(l_buf[B * Hq * Nq:]).all()
    kw = dict(scale=scale, mask_kind=MASK_ID[mask], window=window, softcap=softcap,
              doc_offsets=docs, alibi_slopes=slopes)
    O_ref, L_ref = oracle.attention(f64(q), f64(k), f64(v), **kw)
    bound = None
    if v_std > 1.0:
        # wide V: the derived per-element bound of bf16 rounding (see gpu_common)
        PV_abs, _ = oracle.attention(f64(q), f64(k), np.abs(f64(v)), **kw)
        bound = BF16_UNIT_ROUNDOFF * (np.abs(O_ref) + PV_abs)
    return compare(o, lse, O_ref, L_ref,
                   f"{B}x{Hq}/{Hkv}x{Nq}x{Nk}x{d} {mask} w{window} c{softcap} alibi{slopes}",
                   o_bound=bound)


def test_tiny_workload_noncausal_and_causal():
    w = workloads.TINY
    for mask in ("none", "causal"):
        q, k, v = workloads.make_inputs(w)
        q, k, v = q.cuda(), k.cuda(), v.cuda()
        o, lse = attn_fwd(q, k, v, scale=w.scale, mask=mask)
        assert device_status() == 0
        assert o.shape == (1, 2, 128, 64) and lse.shape == (1, 2, 128)
        O_ref, L_ref = oracle.attention(f64(q), f64(k), f64(v), scale=w.scale,
                                        mask_kind=MASK_ID[mask])
        compare(o, lse, O_ref, L_ref, f"tiny {mask}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 255, 256, 257, 700])
@pytest.mark.parametrize("mask", ["none", "causal"])
def test_ragged_lengths(d, N, mask):
    _run_full(1, 2, 2, N, N, d, mask=mask, seed=N)


@pytest.mark.parametrize("Hq,Hkv", [(4, 1), (8, 2), (6, 3), (2, 1), (9, 3), (3, 1)])
def test_gqa_mqa_head_mapping(Hq, Hkv):
    # even groups run two query heads of a KV group side by side, odd ones two row tiles
    _run_full(2, Hq, Hkv, 300, 300, 128, mask="causal", seed=Hq * 10 + Hkv)


@pytest.mark.parametrize("mask,window,docs,d", [
    ("sliding_causal", 200, None, 128), ("document_causal", 0, [0, 130, 131, 500, 777], 128),
    ("none", 0, None, 64), ("sliding", 90, None, 64)])
def test_gqa_head_pairs_under_every_mask(mask, window, docs, d):
    _run_full(2, 8, 2, 777, 777, d, mask=mask, window=window, docs=docs, seed=window + d)


@pytest.mark.parametrize("window", [0, 1, 100, 127, 128, 129, 255, 600])
def test_sliding_window(window):
    _run_full(1, 2, 1, 777, 777, 128, mask="sliding_causal", window=window, seed=window)


@pytest.mark.parametrize("docs", [[0, 1000], [0, 1, 2, 3, 1000], [0, 127, 128, 129, 384, 700, 1000],
                                  [0, 300, 301, 555, 1000]])
def test_document_mask(docs):
    _run_full(1, 3, 3, 1000, 1000, 128, mask="document_causal", docs=docs, seed=len(docs))


@pytest.mark.parametrize("mask", ["none", "causal", "document_causal"])
def test_softcap(mask):
    docs = [0, 200, 513, 800] if mask == "document_causal" else None
    # the packed-document workload's inputs: Q, K and V all N(0,1) * 2
    _run_full(1, 2, 2, 800, 800, 128, mask=mask, softcap=50.0, docs=docs, seed=3, std=2.0,
              v_std=2.0)
    _run_full(1, 2, 2, 300, 300, 64, mask=mask if mask != "document_causal" else "causal",
              softcap=5.0, seed=4, std=3.0)
    # cap 10 with std-2 inputs: |scale s / cap| ~ 0.4, so rows above and below the
    # polynomial tanh's range of 1 mix inside every warp
    _run_full(1, 2, 2, 520, 520, 128, mask=mask, softcap=10.0, docs=docs, seed=5, std=2.0)
    # a small cap (0.5) on small scores: the polynomial path with cap_log2 < 1, where the
    # masked columns' stand-in score must still give exponentials of exactly 0
    _run_full(1, 2, 2, 520, 520, 128, mask=mask, softcap=0.5, docs=docs, seed=6, std=0.2)


@pytest.mark.parametrize("Nq,Nk", [(1, 300), (100, 1000), (300, 129), (513, 64)])
def test_non_square_unmasked(Nq, Nk):
    _run_full(2, 2, 1, Nq, Nk, 128, seed=Nq + Nk)


def test_explicit_scale_and_large_values():
    _run_full(1, 2, 2, 400, 400, 128, mask="causal", scale=0.3, std=3.0, seed=9)


def test_no_keys_gives_zero_and_minus_inf():
    q, k, v = _inputs(1, 2, 2, 10, 1, 64, 1)
    o, lse = attn_fwd(q, k[:, :, :0].contiguous(), v[:, :, :0].contiguous())
    assert device_status() == 0
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_empty_batch_is_a_noop():
    q = torch.empty((0, 2, 8, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = attn_fwd(q, q, q)
    assert o.shape == (0, 2, 8, 64)


def test_unsupported_raises_instead_of_falling_back():
    q, k, v = _inputs(1, 2, 2, 8, 8, 64, 2)
    q96 = torch.zeros((1, 2, 8, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError, match="unsupported"):
        attn_fwd(q96, q96, q96)
    with pytest.raises(RuntimeError, match="unsupported"):
        attn_fwd(q, k[:, :, :4].contiguous(), v[:, :, :4].contiguous(), mask="causal")


# ------------------------------------------------------------------ full-size workloads

def _sampled_full_size(w: workloads.Workload, n_heads: int = 3, seed: int = 0):
    q, k, v = workloads.make_inputs(w, device="cuda")
    docs = workloads.workload_doc_offsets(w)
    doc_t = None if docs is None else torch.tensor(docs, dtype=torch.int32, device="cuda")
    o, lse = attn_fwd(q, k, v, scale=w.scale, mask=w.mask_kind, window=w.window,
                      softcap=w.softcap, doc_offsets=doc_t)
    assert device_status() == 0
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(seed)
    G = w.Hq // w.Hkv
    pairs = {(0, 0), (w.B - 1, w.Hq - 1)}
    while len(pairs) < n_heads + 2:
        pairs.add((int(rng.integers(w.B)), int(rng.integers(w.Hq))))
    for b, h in sorted(pairs):
        rows = sample_rows(w.Nq, rng)
        K = f64(k[b, h // G])
        V = f64(v[b, h // G])
        O_ref, L_ref = oracle.attention_head(f64(q[b, h, rows]), rows, K, V, w.scale,
                                             w.mask_kind, w.window, w.softcap, docs)
        compare(o[b, h, rows], lse[b, h, rows], O_ref, L_ref, f"{w.name} b{b} h{h}")


def test_causal_mha_full_size_sampled():
    _sampled_full_size(workloads.CAUSAL_MHA)


def test_sliding_gqa_full_size_sampled():
    _sampled_full_size(workloads.SWA_GQA)


def test_document_softcap_full_size_sampled():
    _sampled_full_size(workloads.DOC_SOFTCAP)


def test_repeated_calls_are_deterministic():
    q, k, v = _inputs(2, 4, 2, 1000, 1000, 128, 11)
    o1, l1 = attn_fwd(q, k, v, mask="causal")
    o2, l2 = attn_fwd(q, k, v, mask="causal")
    assert device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("window", [0, 1, 63, 127, 128, 129, 300, 2000])
@pytest.mark.parametrize("N", [129, 777])
def test_symmetric_sliding_window(window, N):
    _run_full(1, 2, 1, N, N, 128, mask="sliding", window=window, seed=window + N)


def test_symmetric_sliding_window_d64_gqa():
    _run_full(2, 6, 2, 513, 513, 64, mask="sliding", window=200, seed=5)


def _alibi_slopes(H):
    # the usual geometric ALiBi slopes 2^(-8 (h + 1) / H)
    return [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]


@pytest.mark.parametrize("mask,window", [("none", 0), ("causal", 0), ("sliding_causal", 100),
                                         ("sliding", 100), ("document_causal", 0)])
@pytest.mark.parametrize("d", [64, 128])
def test_alibi_bias(mask, window, d):
    docs = [0, 130, 131, 400, 700] if mask == "document_causal" else None
    _run_full(1, 4, 2, 700, 700, d, mask=mask, window=window, docs=docs, seed=7,
              slopes=_alibi_slopes(4))


@pytest.mark.parametrize("N", [1, 127, 128, 129, 257])
def test_alibi_ragged_and_steep_slopes(N):
    # slope 4: each step back in distance divides the weight by e^4; slope 0 is plain attention
    _run_full(1, 3, 3, N, N, 128, mask="causal", seed=N, slopes=[4.0, 0.0, 0.03125])
    _run_full(1, 2, 1, N, N, 128, mask="none", seed=N + 1, slopes=[1.0, 0.001])


def test_alibi_full_size_sampled():
    # causal MHA workload shapes (B=8, H=32, N=4096, d=128) with geometric slopes, sampled rows
    w = workloads.CAUSAL_MHA
    q, k, v = workloads.make_inputs(w, device="cuda")
    slopes = torch.tensor(_alibi_slopes(w.Hq), dtype=torch.float32, device="cuda")
    o, lse = attn_fwd(q, k, v, scale=w.scale, mask="causal", alibi_slopes=slopes)
    assert device_status() == 0
    rng = np.random.default_rng(5)
    for b, h in [(0, 0), (7, 31), (3, 17)]:
        rows = sample_rows(w.Nq, rng, 24)
        O_ref, L_ref = oracle.attention_head(f64(q[b, h, rows]), rows, f64(k[b, h]), f64(v[b, h]),
                                             w.scale, 1, alibi_slope=float(slopes[h]))
        compare(o[b, h, rows], lse[b, h, rows], O_ref, L_ref, f"alibi full b{b} h{h}")


def test_alibi_with_softcap_is_unsupported():
    q, k, v = _inputs(1, 2, 2, 64, 64, 128, 1)
    slopes = torch.tensor([0.5, 0.25], dtype=torch.float32, device="cuda")
    with pytest.raises(Exception) as e:
        attn_fwd(q, k, v, mask="causal", softcap=30.0, alibi_slopes=slopes)
    assert "unsupported" in str(e.value).lower()
