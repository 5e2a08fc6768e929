"""Parity of the backward pass (attn_bwd through the C ABI) with the fp64 oracle's gradients.

The kernels take attn_fwd's bf16 O and fp32 LSE and round P and dS to bf16 for the tensor
core, as the forward pass rounds P; dQ, dK, dV are rounded to bf16.  The oracle's gradients
are exact (fp64 from the same bf16 inputs).  Errors are measured relative to the size of
each gradient tensor: the largest error against the largest |reference| and the mean error
against the mean |reference|."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from io_aware_softmax_b200 import attn_bwd, attn_fwd, device_status
from tests.gpu_common import f64

pytestmark = pytest.mark.gpu

MASK_ID = {"none": 0, "causal": 1, "sliding_causal": 2, "document_causal": 3, "sliding": 4}
# Relative bounds: rounding P, dS and the outputs to bf16 costs up to 2^-9 relative per
# element each, so the mean error is about 2^-9 of the mean gradient (measured: 1.8e-3 to
# 2.9e-3) and the worst element a few such roundings (measured: at most 5.4e-3 of the largest
# gradient): bounds 2^-8 on the mean and about 4 x 2^-8 on the maximum.  A reference that is
# identically zero (one key: the softmax Jacobian vanishes) is compared against absolute
# floors: 1e-3 for the maximum, 1e-4 for the mean.
TOL_MAX = 1.5e-2
TOL_MEAN = 4e-3


def compare_grad(got, ref, what, tol_mean=TOL_MEAN):
    g = f64(got)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    err = np.abs(g - ref)
    big = max(float(np.abs(ref).max()), 1e-3)
    avg = max(float(np.abs(ref).mean()), 1e-4)
    rmax, rmean = float(err.max()) / big, float(err.mean()) / avg
    print(f"{what}: max {rmax:.2e} of max|ref|, mean {rmean:.2e} of mean|ref|")
    assert rmax <= TOL_MAX and rmean <= tol_mean, f"{what}: max {rmax:.3e}, mean {rmean:.3e}"


def _run(B, Hq, Hkv, Nq, Nk, d, mask="none", window=0, docs=None, seed=0, scale=None,
         slopes=None, softcap=0.0, std=1.0, tol_mean=TOL_MEAN):
    q = workloads.randn_bf16((B, Hq, Nq, d), seed, 0, std).cuda()
    k = workloads.randn_bf16((B, Hkv, Nk, d), seed, 1, std).cuda()
    v = workloads.randn_bf16((B, Hkv, Nk, d), seed, 2).cuda()
    dout = workloads.randn_bf16((B, Hq, Nq, d), seed, 3).cuda()
    doc_t = None if docs is None else torch.tensor(docs, dtype=torch.int32, device="cuda")
    slopes_t = None if slopes is None else torch.tensor(slopes, dtype=torch.float32, device="cuda")
    o, lse = attn_fwd(q, k, v, scale=scale, mask=mask, window=window, doc_offsets=doc_t,
                      alibi_slopes=slopes_t, softcap=softcap)
    dq, dk, dv = attn_bwd(q, k, v, o, lse, dout, scale=scale, mask=mask, window=window,
                          doc_offsets=doc_t, alibi_slopes=slopes_t, softcap=softcap)
    assert device_status() == 0
    rq, rk, rv = oracle.attention_backward(f64(q), f64(k), f64(v), f64(dout), scale=scale,
                                           mask_kind=MASK_ID[mask], window=window,
                                           doc_offsets=docs, alibi_slopes=slopes,
                                           softcap=softcap)
    tag = (f"{B}x{Hq}/{Hkv}x{Nq}x{Nk}x{d} {mask} w{window}"
           + ("" if slopes is None else " alibi") + (f" cap{softcap}" if softcap else ""))
    compare_grad(dq, rq, "dQ " + tag, tol_mean)
    compare_grad(dk, rk, "dK " + tag, tol_mean)
    compare_grad(dv, rv, "dV " + tag, tol_mean)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 300])
@pytest.mark.parametrize("mask", ["none", "causal"])
def test_ragged_lengths(d, N, mask):
    _run(1, 2, 2, N, N, d, mask=mask, seed=N + d)


@pytest.mark.parametrize("Hq,Hkv", [(4, 1), (8, 2), (6, 3)])
def test_gqa_sums_over_the_group(Hq, Hkv):
    _run(2, Hq, Hkv, 300, 300, 128, mask="causal", seed=Hq * 10 + Hkv)


@pytest.mark.parametrize("mask,window", [("sliding_causal", 100), ("sliding_causal", 0),
                                         ("sliding", 130), ("sliding", 1)])
def test_windows(mask, window):
    _run(1, 2, 1, 700, 700, 128, mask=mask, window=window, seed=window + 3)


def test_document_mask():
    _run(1, 3, 3, 800, 800, 128, mask="document_causal", docs=[0, 1, 127, 300, 301, 700, 800],
         seed=8)


@pytest.mark.parametrize("Nq,Nk", [(100, 300), (300, 129), (1, 200)])
def test_non_square_unmasked(Nq, Nk):
    _run(1, 2, 1, Nq, Nk, 128, seed=Nq + Nk, scale=0.2)


def _geometric_slopes(H):
    return [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]


@pytest.mark.parametrize("mask,N,d", [("causal", 300, 128), ("none", 257, 64),
                                      ("sliding", 700, 128)])
def test_alibi(mask, N, d):
    # GQA (4 query heads on 2 KV heads): the dK/dV kernel takes each streamed tile's slope
    _run(1, 4, 2, N, N, d, mask=mask, window=130, seed=N + d, slopes=_geometric_slopes(4))


def test_alibi_steep_slopes_and_ragged_tail():
    # Slope 2: the bias dominates the scores and the diagonal key carries P_max ~ 0.86 of
    # every row (weights 1, e^-2, e^-4, ...).  dS = P (dP - D) then cancels: D = rowsum(dO O)
    # is taken from the forward's stored bf16 O (2^-9 relative per element), and dP - D is
    # only about (1 - P_max) of dP, so D's rounding reaches dS amplified by 1 / (1 - P_max)
    # ~ 7 on that head.  Averaged with the diffuse second head (slope 0.03) the mean error
    # bound becomes 2^-7 of the mean gradient; the maximum keeps its bound.
    _run(2, 2, 1, 129, 129, 128, mask="causal", seed=21, slopes=[2.0, 0.03], tol_mean=2.0 ** -7)


@pytest.mark.parametrize("mask,N,d,cap,std", [("causal", 300, 128, 1.5, 1.0),
                                               ("none", 129, 64, 3.0, 2.0),
                                               ("sliding", 700, 128, 1.0, 1.0)])
def test_softcap(mask, N, d, cap, std):
    # small caps saturate many scores, so the (1 - tanh^2) factor matters
    _run(1, 4, 2, N, N, d, mask=mask, window=130, seed=N + d, softcap=cap, std=std)


def test_document_softcap_as_the_packed_workload():
    # the packed-document workload's hooks (cap 50, inputs N(0,1) * 2) on short documents
    _run(1, 3, 3, 800, 800, 128, mask="document_causal", docs=[0, 1, 127, 300, 301, 700, 800],
         seed=9, softcap=50.0, std=2.0)


def test_alibi_with_softcap_is_unsupported():
    q = workloads.randn_bf16((1, 2, 64, 128), 1, 0).cuda()
    slopes = torch.tensor([0.5, 0.25], dtype=torch.float32, device="cuda")
    lse = torch.zeros((1, 2, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(Exception) as e:
        attn_bwd(q, q, q, q, lse, q, alibi_slopes=slopes, softcap=30.0)
    assert "unsupported" in str(e.value).lower()


def test_causal_mha_full_size_one_head():
    # the causal MHA workload (B=8, H=32, N=4096, d=128): gradients of head (b=5, h=19)
    # against the oracle over all 4096 rows
    w = workloads.CAUSAL_MHA
    q, k, v = workloads.make_inputs(w, device="cuda")
    dout = workloads.randn_bf16((w.B, w.Hq, w.Nq, w.d), w.seed, 3, device="cuda")
    o, lse = attn_fwd(q, k, v, scale=w.scale, mask="causal")
    dq, dk, dv = attn_bwd(q, k, v, o, lse, dout, scale=w.scale, mask="causal")
    assert device_status() == 0
    b, h = 5, 19
    sl = lambda t: f64(t[b:b + 1, h:h + 1])
    rq, rk, rv = oracle.attention_backward(sl(q), sl(k), sl(v), sl(dout), scale=w.scale,
                                           mask_kind=1)
    compare_grad(dq[b:b + 1, h:h + 1], rq, "dQ full")
    compare_grad(dk[b:b + 1, h:h + 1], rk, "dK full")
    compare_grad(dv[b:b + 1, h:h + 1], rv, "dV full")
