"""FP8 (E4M3) path: the block quantizer and attn_fwd_fp8 against the oracle (fp8 module).

The attention oracle is exact attention of the dequantized codes the quantizer produced, so
the kernel's remaining error is P rounded to E4M3 before the P V product (at most 2^-4
relative per element in E4M3's normal range, which the 64 P scaling keeps probabilities
down to 2^-12 of the row max in) and O rounded to bf16.  Bounds: the maximum O error at most
2^-5 of max |V| (each output is a convex combination of V rows, each weight off by at most
2^-4 relative; see TOL_MAX_O), the mean O error 2^-7 of the mean |V| (round-to-nearest leaves 2^-5 relative
on average per weight, and the signs of those errors vary over the visible keys of a row;
measured at most 4.7e-3), and LSE within 1e-3 (it comes from the fp32 P, not the rounded
one; measured at most 2.6e-6)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from io_aware_softmax_b200 import attn_fwd_fp8, device_status, quantize_fp8
from oracle import fp8 as ofp8
from tests.gpu_common import f64

pytestmark = pytest.mark.gpu

MASK_ID = {"none": 0, "causal": 1, "sliding_causal": 2, "document_causal": 3, "sliding": 4}
TOL_MEAN_O = 2.0 ** -7
# 2^-4 of max|V| is the worst case (every weight rounded the same way by the full 2^-4);
# rounding errors of different weights have different signs, and the largest weight of a
# row (P = 1 at the reference max, 64 in E4M3) is exact, so the measured maximum stays at
# or below 0.020 of max|V| over every case here.  The bound is 2^-5, which a doubling of the
# worst measured error would exceed.
TOL_MAX_O = 2.0 ** -5


def _codes(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 127, 300])
def test_quantizer_is_bit_exact_without_rotation(d, N):
    x = (workloads.randn_bf16((2, 3, N, d), N + d, 0).float()
         * torch.tensor([1.0, 30.0, 0.02]).view(1, 3, 1, 1)).to(torch.bfloat16)
    x[1, 2, :min(N, 128)] = 0                               # an all-zero first block
    codes, scales = quantize_fp8(x.cuda(), block_rows=128)
    assert device_status() == 0
    want_c, want_s = ofp8.quantize_blocks(x.float().numpy(), 128)
    assert np.array_equal(_codes(codes), want_c)
    assert np.allclose(scales.cpu().numpy(), want_s, rtol=1e-6, atol=0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,n_pad", [(300, 304), (128, 144), (5, 16), (2100, 2112),
                                     (130, 400), (1100, 1424)])
def test_quantizer_transposed_per_head(d, N, n_pad):
    # one scale per head (the V layout of attn_fwd_fp8): a cluster of CTAs per head; more
    # sub-blocks of 128 keys than CTAs (2100), and n_pad reaching past the last sub-block
    # with keys (130 -> 400, 1100 -> 1424), whose columns must come out zero
    x = workloads.randn_bf16((2, 2, N, d), N + d, 1)
    codes, scales = quantize_fp8(x.cuda(), block_rows=N, transpose=True, n_pad=n_pad)
    assert device_status() == 0
    assert codes.shape == (2, 2, d, n_pad) and scales.shape == (2, 2, 1)
    want_c, want_s = ofp8.quantize_blocks(x.float().numpy(), N)
    got = _codes(codes)
    assert np.array_equal(got[..., :N], np.swapaxes(want_c, 2, 3))
    assert np.all(got[..., N:] == 0.0)
    assert np.allclose(scales.cpu().numpy(), want_s, rtol=1e-6, atol=0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,block_rows,transpose", [(700, 300, False), (700, 700, False),
                                                    (300, 64, True), (130, 7, True),
                                                    (100, 3, False), (500, 64, False),
                                                    (333, 100, False), (129, 16, False)])
def test_quantizer_blocks_are_bit_exact(d, N, block_rows, transpose):
    # row-major blocks of at most 128 rows (a tiled copy of block_rows rows each, ragged last
    # blocks), blocks longer than 128 rows, and transposed outputs with several blocks per
    # head (the chunked amax / codes / finalize launches)
    x = (workloads.randn_bf16((2, 2, N, d), N + block_rows, 3).float()
         * torch.tensor([1.0, 7.0]).view(1, 2, 1, 1)).to(torch.bfloat16)
    n_pad = -(-N // 16) * 16
    codes, scales = quantize_fp8(x.cuda(), block_rows=block_rows, transpose=transpose,
                                 n_pad=n_pad if transpose else None)
    assert device_status() == 0
    want_c, want_s = ofp8.quantize_blocks(x.float().numpy(), block_rows)
    got = _codes(codes)
    if transpose:
        assert np.array_equal(got[..., :N], np.swapaxes(want_c, 2, 3))
        assert np.all(got[..., N:] == 0.0)
    else:
        assert np.array_equal(got, want_c)
    assert np.allclose(scales.cpu().numpy(), want_s, rtol=1e-6, atol=0)


@pytest.mark.parametrize("d", [64, 128])
def test_quantizer_row_major_output_aligned_to_4_bytes(d):
    # a row-major output that is 4-byte but not 16-byte aligned takes 4-byte stores
    from io_aware_softmax_b200 import _lib
    N = 300
    x = workloads.randn_bf16((1, 2, N, d), 77, 4).cuda()
    buf = torch.zeros(2 * N * d + 64, dtype=torch.uint8, device="cuda")
    scales = torch.empty((1, 2, 3), dtype=torch.float32, device="cuda")
    st = _lib.load().attn_quantize_fp8(x.data_ptr(), buf.data_ptr() + 4, scales.data_ptr(), 1, 2,
                                       N, d, 128, 0, 0, None,
                                       torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0 and device_status() == 0
    got = buf[4:4 + 2 * N * d].view(torch.float8_e4m3fn).float().cpu().numpy().reshape(1, 2, N, d)
    want_c, want_s = ofp8.quantize_blocks(x.cpu().float().numpy(), 128)
    assert np.array_equal(got.astype(np.float64), want_c)
    assert torch.all(buf[:4] == 0) and torch.all(buf[4 + 2 * N * d:] == 0)   # nothing outside
    assert np.allclose(scales.cpu().numpy(), want_s, rtol=1e-6, atol=0)


@pytest.mark.parametrize("d", [64, 128])
def test_rotated_codes_agree_between_kernels(d):
    # rotation in one thread's registers (row-major, 128-row blocks) and across lanes
    # (transposed blocks of 128 rows) round every operation alike: the same bits
    x = workloads.randn_bf16((2, 2, 300, d), 5 * d, 5)
    x[0, 1, :, 3] *= 50
    signs = torch.from_numpy(np.random.default_rng(d + 1).choice([-1.0, 1.0], d)
                             .astype(np.float32)).cuda()
    c_row, s_row = quantize_fp8(x.cuda(), block_rows=128, signs=signs)
    c_t, s_t = quantize_fp8(x.cuda(), block_rows=128, signs=signs, transpose=True, n_pad=304)
    assert device_status() == 0
    assert torch.equal(s_row, s_t)
    assert torch.equal(c_row.view(torch.uint8),
                       c_t.view(torch.uint8)[..., :300].transpose(2, 3))


@pytest.mark.parametrize("d", [64, 128])
def test_quantizer_rotation_within_e4m3_rounding(d):
    x = workloads.randn_bf16((1, 2, 260, d), d, 2)
    x[0, 0, :, 5] *= 40                                     # an outlier column
    signs = torch.from_numpy(np.random.default_rng(d).choice([-1.0, 1.0], d).astype(np.float32))
    codes, scales = quantize_fp8(x.cuda(), block_rows=128, signs=signs.cuda())
    assert device_status() == 0
    rot = ofp8.rotate(x.float().numpy(), signs.numpy())
    deq = ofp8.dequantize_blocks(_codes(codes), scales.cpu().numpy(), 128)
    rep = np.repeat(scales.cpu().numpy(), 128, axis=2)[:, :, :260, None]
    assert np.all(np.abs(deq - rot) <= 2 ** -4 * np.abs(rot) + rep * 2 ** -10 + 1e-5 * np.abs(rot).max())
    # the rotation spread the outlier: the head's scale is far below the unrotated one
    _, s_plain = quantize_fp8(x.cuda(), block_rows=128)
    assert float(scales[0, 0, 0]) < 0.4 * float(s_plain[0, 0, 0])


def _fp8_case(B, Hq, Hkv, N, mask="none", window=0, docs=None, seed=0, rotate=True, std=1.0):
    d = 128
    q = workloads.randn_bf16((B, Hq, N, d), seed, 0, std).cuda()
    k = workloads.randn_bf16((B, Hkv, N, d), seed, 1, std).cuda()
    v = workloads.randn_bf16((B, Hkv, N, d), seed, 2, std).cuda()
    signs = None
    if rotate:
        rng = np.random.default_rng(seed)
        signs = torch.from_numpy(rng.choice([-1.0, 1.0], d).astype(np.float32)).cuda()
    q8, qs = quantize_fp8(q, block_rows=128, signs=signs)
    k8, ks = quantize_fp8(k, block_rows=128, signs=signs)
    vt8, vs = quantize_fp8(v, block_rows=N, transpose=True)
    doc_t = None if docs is None else torch.tensor(docs, dtype=torch.int32, device="cuda")
    o, lse = attn_fwd_fp8(q8, qs, k8, ks, vt8, vs[:, :, 0], mask=mask, window=window,
                          doc_offsets=doc_t)
    assert device_status() == 0
    vcodes = np.swapaxes(_codes(vt8)[..., :N], 2, 3)
    O_ref, L_ref = ofp8.attention_fp8(_codes(q8), qs.cpu().numpy(), _codes(k8),
                                      ks.cpu().numpy(), vcodes, vs.cpu().numpy()[:, :, 0],
                                      mask_kind=MASK_ID[mask], window=window, doc_offsets=docs)
    O = f64(o)
    vmax = float(np.abs(vcodes * vs.cpu().numpy()[:, :, 0][:, :, None, None]).max())
    vmean = float(np.abs(vcodes * vs.cpu().numpy()[:, :, 0][:, :, None, None]).mean())
    err = np.abs(O - O_ref)
    lerr = np.abs(f64(lse) - L_ref)
    tag = f"fp8 {B}x{Hq}/{Hkv}x{N} {mask} w{window} rot{rotate}"
    print(f"{tag}: O max {err.max() / vmax:.2e} of max|V|, mean {err.mean() / vmean:.2e} of "
          f"mean|V|, LSE max {lerr.max():.2e}")
    assert np.all(np.isfinite(O))
    assert err.max() <= TOL_MAX_O * vmax, tag
    assert err.mean() <= TOL_MEAN_O * vmean, tag
    assert lerr.max() <= 1e-3, tag


@pytest.mark.parametrize("N", [1, 129, 300, 777])
@pytest.mark.parametrize("mask", ["none", "causal"])
def test_fp8_attention_ragged(N, mask):
    _fp8_case(1, 2, 2, N, mask=mask, seed=N)


def test_fp8_attention_gqa_and_no_rotation():
    _fp8_case(2, 8, 2, 600, mask="causal", seed=3)
    _fp8_case(1, 4, 1, 600, mask="causal", seed=4, rotate=False)


@pytest.mark.parametrize("mask,window,docs", [("sliding_causal", 100, None), ("sliding", 70, None),
                                              ("document_causal", 0, [0, 100, 101, 700, 900])])
def test_fp8_attention_masks(mask, window, docs):
    _fp8_case(1, 2, 1, 900, mask=mask, window=window, docs=docs, seed=window + 11)


def test_fp8_attention_large_scores():
    _fp8_case(1, 2, 2, 500, mask="causal", seed=12, std=2.5)


def test_fp8_head_dim_64_is_unsupported():
    q8 = torch.zeros((1, 1, 8, 64), dtype=torch.float8_e4m3fn, device="cuda")
    vt8 = torch.zeros((1, 1, 64, 16), dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.ones((1, 1, 1), dtype=torch.float32, device="cuda")
    with pytest.raises(Exception) as e:
        attn_fwd_fp8(q8, s, q8, s, vt8, s[:, :, 0])
    assert "unsupported" in str(e.value).lower()


def _outlier_inputs(B, H, N, d, seed, frac=1e-3, mag=10.0):
    # N(0,1) with a fraction `frac` of the entries of Q and K replaced by N(0, mag^2): the
    # outliers whose effect the rotation is meant to spread
    gen = torch.Generator().manual_seed(seed)
    q, k, v = (workloads.randn_bf16((B, H, N, d), seed, i) for i in range(3))
    for t in (q, k):
        hit = torch.rand(t.shape, generator=gen) < frac
        t[hit] = (torch.randn(int(hit.sum()), generator=gen) * mag).to(torch.bfloat16)
    return q.cuda(), k.cuda(), v.cuda()


def _fp8_vs_exact(q, k, v, rotate, seed):
    B, H, N, d = q.shape
    signs = None
    if rotate:
        signs = torch.from_numpy(np.random.default_rng(seed).choice([-1.0, 1.0], d)
                                 .astype(np.float32)).cuda()
    q8, qs = quantize_fp8(q, block_rows=128, signs=signs)
    k8, ks = quantize_fp8(k, block_rows=128, signs=signs)
    vt8, vs = quantize_fp8(v, block_rows=N, transpose=True)
    o, lse = attn_fwd_fp8(q8, qs, k8, ks, vt8, vs[:, :, 0].contiguous(), mask="causal")
    assert device_status() == 0
    O_ref, L_ref = oracle.attention(f64(q), f64(k), f64(v), mask_kind=1)
    err = f64(o) - O_ref
    return (float(np.sqrt(np.mean(err ** 2))), float(np.abs(err).max()),
            float(np.abs(f64(lse) - L_ref).max()))


def test_fp8_accuracy_against_the_unquantized_inputs():
    # The pages credit block quantization plus incoherent processing with keeping FP8
    # attention accurate ("FP8 지원과 정확도 유지").  Against exact attention of the original
    # bf16 inputs (not of the dequantized codes), on inputs with outlier entries (0.1 % of
    # Q and K drawn with std 10): the rotated path must be more accurate than the plain one
    # in every measure.  Measured on this input: rotated rmse 9.1e-3, max 0.20, LSE 0.17;
    # plain 1.2e-2, 0.44, 1.15.  The absolute bounds below sit about 1.5x above the rotated
    # figures, so a regression of the rotation or the block scales fails them.
    q, k, v = _outlier_inputs(1, 4, 1024, 128, seed=71)
    rot = _fp8_vs_exact(q, k, v, True, 71)
    plain = _fp8_vs_exact(q, k, v, False, 71)
    print(f"fp8 vs exact, outlier inputs: rotated rmse {rot[0]:.2e} max {rot[1]:.2e} "
          f"LSE {rot[2]:.2e}; plain rmse {plain[0]:.2e} max {plain[1]:.2e} LSE {plain[2]:.2e}")
    assert rot[0] < plain[0] and rot[1] < plain[1] and rot[2] < plain[2]
    assert rot[0] <= 1.4e-2 and rot[1] <= 0.3 and rot[2] <= 0.25
