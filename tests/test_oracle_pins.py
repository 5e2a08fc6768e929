"""Pins of the fp64 oracle to facts the pages and the mathematics fix (CPU only).

Each pin is chosen so that a plausible mistake in the oracle -- a dropped scale, a wrong
sign, a transposed operand, an off-by-one in a mask bound, a wrong GQA head mapping, a
log base, a merge weight -- fails at least one of them.  Library special cases use torch's
CPU float64 SDPA with masks built here independently of the oracle's ``visible``.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import (MASK_CAUSAL, MASK_DOCUMENT_CAUSAL, MASK_NONE, MASK_SLIDING,
                    MASK_SLIDING_CAUSAL, TILE_EMPTY, TILE_FULL, TILE_PARTIAL)
import workloads
from workloads import accounting

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    out = []
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append(line)
    return out


def _one_row(scores, scale=1.0):
    """Attention of one query over keys whose scaled scores are ``scores``: q = [1],
    k_j = [s_j], V = identity so that O is the probability row."""
    s = np.asarray(scores, dtype=np.float64)
    q = np.ones((1, 1, 1, 1))
    k = (s / scale).reshape(1, 1, -1, 1)
    v = np.eye(len(s)).reshape(1, 1, len(s), len(s))
    O, lse = oracle.attention(q, k, v, scale=scale)
    return O[0, 0, 0], lse[0, 0, 0]


# --------------------------------------------------------------------- worked examples

def test_worked_softmax_example_figure4():
    for line in _rows("softmax_row_worked_example.txt"):
        name, scores, qty, printed, tol = line.split()
        scores = [float(x) for x in scores.split(",")]
        printed, tol = float(printed), float(tol)
        p, lse = _one_row(scores)
        expsum = math.exp(lse)            # LSE is ln(sum exp(s)) when the max is 0
        if qty == "p0":
            got = p[0]
        elif qty == "expsum":
            got = expsum
        elif qty == "exp2":
            got = (expsum - 2.0) / 2.0    # the two keys of score 2 share the rest
        else:
            raise AssertionError(qty)
        assert abs(got - printed) <= tol + 1e-12, (name, qty, got, printed)
        assert abs(p.sum() - 1.0) < 1e-15


def test_partial_softmax_is_not_the_row_softmax_but_merges_to_it():
    # Figure 4: the first two keys alone give 0.5 each, not 0.25 / ~0.06.
    p_part, lse_a = _one_row([0.0, 0.0])
    p_full, lse_full = _one_row([0.0, 0.0, 2.0, 2.0])
    assert p_part[0] == 0.5 and abs(p_full[0] - 1 / (2 + 2 * math.e ** 2)) < 1e-15
    # the other half, then the rescaling merge of the two partial results
    p_b, lse_b = _one_row([2.0, 2.0])
    o_a = np.concatenate([p_part, [0, 0]])
    o_b = np.concatenate([[0, 0], p_b])
    O, lse = oracle.merge_partials(np.stack([o_a, o_b])[None], np.array([[lse_a, lse_b]]))
    assert np.allclose(O[0], p_full, atol=1e-15, rtol=0)
    assert abs(lse[0] - lse_full) < 1e-14


def test_causal_tile_example_figure3():
    T = 4
    for line in _rows("causal_tile_example.txt"):
        qi, keys = line.split()
        want = sorted(int(x) for x in keys.split(","))
        vis = oracle.visible(int(qi), np.arange(T), MASK_CAUSAL)
        assert sorted(np.nonzero(vis)[0].tolist()) == want
    # The tile (queries 2,3 x keys 0,1) is entirely visible, yet the rows' denominators
    # need keys outside it: the tile alone gives a different probability.
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 1, T, 8))
    k = rng.standard_normal((1, 1, T, 8))
    v = rng.standard_normal((1, 1, T, 8))
    assert oracle.tile_map(1, T, T, MASK_CAUSAL, block_q=2, block_kv=2)[0, 1, 0] == TILE_FULL
    _, lse_full = oracle.attention(q, k, v, mask_kind=MASK_CAUSAL)
    _, lse_tile = oracle.attention_head(q[0, 0, 2:4], np.arange(2, 4), k[0, 0, :2],
                                        v[0, 0, :2], 1 / math.sqrt(8), MASK_CAUSAL)
    assert np.all(lse_tile < lse_full[0, 0, 2:4])


# --------------------------------------------------------------------------- invariants

def _rand_qkv(B, Hq, Hkv, N, d, seed, std=1.0, Nk=None):
    rng = np.random.default_rng(seed)
    Nk = N if Nk is None else Nk
    return (std * rng.standard_normal((B, Hq, N, d)), std * rng.standard_normal((B, Hkv, Nk, d)),
            std * rng.standard_normal((B, Hkv, Nk, d)))


DOCS_SMALL = np.array([0, 5, 6, 13, 20], dtype=np.int32)   # lengths 5, 1, 7, 7
MASKS = [(MASK_NONE, 0, None), (MASK_CAUSAL, 0, None), (MASK_SLIDING_CAUSAL, 3, None),
         (MASK_DOCUMENT_CAUSAL, 0, DOCS_SMALL), (MASK_SLIDING, 3, None)]


@pytest.mark.parametrize("mask_kind,window,docs", MASKS)
def test_rows_sum_to_one_and_masked_probabilities_are_zero(mask_kind, window, docs):
    q, k, v = _rand_qkv(1, 1, 1, 20, 16, 1)
    rows = np.arange(20)
    _, _, P = oracle.attention_head(q[0, 0], rows, k[0, 0], v[0, 0], 0.25, mask_kind, window,
                                    0.0, docs, return_probs=True)
    assert np.all(np.abs(P.sum(axis=1) - 1.0) < 1e-12)
    vis = oracle.visible(rows[:, None], rows[None, :], mask_kind, window, docs)
    assert np.all(P[~vis] == 0.0)
    assert np.all(P[vis] > 0.0)


def _visible_counts_by_hand(N, mask_kind, window, docs):
    """Number of keys each query row sees, by counting the definition's interval."""
    out = []
    for i in range(N):
        if mask_kind == MASK_NONE:
            out.append(N)
        elif mask_kind == MASK_CAUSAL:
            out.append(i + 1)
        elif mask_kind == MASK_SLIDING_CAUSAL:
            out.append(min(i, window) + 1)
        elif mask_kind == MASK_SLIDING:
            out.append(min(N - 1, i + window) - max(0, i - window) + 1)
        else:
            start = max(int(o) for o in docs if o <= i)
            out.append(i - start + 1)
    return out


@pytest.mark.parametrize("mask_kind,window,docs", MASKS)
def test_equal_scores_give_mean_of_visible_values(mask_kind, window, docs):
    N, d = 20, 8
    _, k, v = _rand_qkv(1, 1, 1, N, d, 2)
    q = np.zeros((1, 1, N, d))                   # every score 0
    O, lse = oracle.attention(q, k, v, mask_kind=mask_kind, window=window, doc_offsets=docs)
    counts = _visible_counts_by_hand(N, mask_kind, window, docs)
    for i in range(N):
        if mask_kind == MASK_NONE:
            lo, hi = 0, N
        elif mask_kind == MASK_CAUSAL:
            lo, hi = 0, i + 1
        elif mask_kind == MASK_SLIDING_CAUSAL:
            lo, hi = max(0, i - window), i + 1
        elif mask_kind == MASK_SLIDING:
            lo, hi = max(0, i - window), min(N, i + window + 1)
        else:
            lo, hi = max(int(o) for o in docs if o <= i), i + 1
        assert hi - lo == counts[i]
        assert np.allclose(O[0, 0, i], v[0, 0, lo:hi].mean(axis=0), atol=1e-14, rtol=0)
        assert abs(lse[0, 0, i] - math.log(counts[i])) < 1e-14


def test_causal_row0_returns_v0_and_its_own_score():
    q, k, v = _rand_qkv(2, 4, 2, 9, 16, 3)
    scale = 0.3
    O, lse = oracle.attention(q, k, v, scale=scale, mask_kind=MASK_CAUSAL)
    for b in range(2):
        for h in range(4):
            hk = h // 2
            assert np.array_equal(O[b, h, 0], v[b, hk, 0])
            s00 = scale * float(np.dot(q[b, h, 0], k[b, hk, 0]))
            assert abs(lse[b, h, 0] - s00) < 1e-13


# ------------------------------------------------------------- library special cases

def _torch_mask(N, mask_kind, window, docs):
    m = torch.ones(N, N, dtype=torch.bool)
    if mask_kind in (MASK_CAUSAL, MASK_SLIDING_CAUSAL, MASK_DOCUMENT_CAUSAL):
        m = torch.tril(m)
    if mask_kind == MASK_SLIDING_CAUSAL:
        m = m & torch.triu(torch.ones(N, N, dtype=torch.bool), diagonal=-window)
    if mask_kind == MASK_SLIDING:
        m = torch.triu(m, diagonal=-window) & torch.tril(m, diagonal=window)
    if mask_kind == MASK_DOCUMENT_CAUSAL:
        blk = torch.zeros(N, N, dtype=torch.bool)
        for s, e in zip(docs[:-1], docs[1:]):
            blk[s:e, s:e] = True
        m = m & blk
    return m


@pytest.mark.parametrize("mask_kind,window,docs", MASKS)
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (6, 1)])
def test_matches_torch_sdpa_float64(mask_kind, window, docs, Hq, Hkv):
    B, N, d = 2, 20, 16
    q, k, v = _rand_qkv(B, Hq, Hkv, N, d, 4)
    scale = 0.17
    O, lse = oracle.attention(q, k, v, scale=scale, mask_kind=mask_kind, window=window,
                              doc_offsets=docs)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    G = Hq // Hkv
    tk = tk.repeat_interleave(G, dim=1)
    tv = tv.repeat_interleave(G, dim=1)
    if mask_kind == MASK_CAUSAL:
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                               scale=scale)
    else:
        ref = torch.nn.functional.scaled_dot_product_attention(
            tq, tk, tv, attn_mask=_torch_mask(N, mask_kind, window, docs), scale=scale)
    # fp64 on both sides.  In isolation the two agree to 1e-15; inside the full CPU suite
    # torch's CPU kernels now and then differ by up to 7.2e-10 on the first case.  The
    # bound 1e-8 is five orders below the kernels' LSE tolerance and far below the effect
    # of any plausible mistake in the oracle.
    assert np.allclose(O, ref.numpy(), atol=1e-8, rtol=0)
    S = torch.einsum("bhid,bhjd->bhij", tq, tk) * scale
    S = S.masked_fill(~_torch_mask(N, mask_kind, window, docs), float("-inf"))
    assert np.allclose(lse, torch.logsumexp(S, dim=-1).numpy(), atol=1e-8, rtol=0)


def test_non_square_unmasked_and_default_scale():
    q, k, v = _rand_qkv(1, 2, 2, 3, 32, 5, Nk=11)
    O, lse = oracle.attention(q, k, v)            # scale None -> 1/sqrt(d)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x) for x in (q, k, v)))
    assert np.allclose(O, ref.numpy(), atol=1e-8, rtol=0)


# ------------------------------------------------------------------------------ soft-cap

def test_softcap_limits():
    q, k, v = _rand_qkv(1, 2, 1, 16, 8, 6, std=3.0)
    O0, l0 = oracle.attention(q, k, v, mask_kind=MASK_CAUSAL)
    O1, l1 = oracle.attention(q, k, v, mask_kind=MASK_CAUSAL, softcap=1e9)
    assert np.allclose(O0, O1, atol=1e-12) and np.allclose(l0, l1, atol=1e-12)
    s = np.linspace(-500, 500, 101)
    c = oracle.softcap_scores(s, 50.0)
    assert np.all(np.abs(c) < 50.0) and np.allclose(c, -oracle.softcap_scores(-s, 50.0))
    assert abs(oracle.softcap_scores(np.array([1e4]), 50.0)[0] - 50.0) < 1e-12
    assert np.all(np.diff(c) > 0)


def test_softcap_acts_on_the_scaled_score():
    # one visible key: LSE equals the (capped) score itself.  q.k = 100, scale 0.5 ->
    # scaled score 50; capped at c = 50: 50 * tanh(1) = 38.0797...
    q = np.array([10.0]).reshape(1, 1, 1, 1)
    k = np.array([10.0]).reshape(1, 1, 1, 1)
    v = np.ones((1, 1, 1, 1))
    _, lse = oracle.attention(q, k, v, scale=0.5, softcap=50.0)
    assert abs(lse[0, 0, 0] - 38.07970779778824) < 1e-12


# ---------------------------------------------------------------- tiled and split merges

@pytest.mark.parametrize("mask_kind,window,docs", MASKS)
@pytest.mark.parametrize("bq,bk", [(1, 1), (2, 3), (3, 7), (5, 2), (16, 16)])
def test_tiled_online_softmax_equals_full(mask_kind, window, docs, bq, bk):
    q, k, v = _rand_qkv(1, 2, 1, 20, 8, 7, std=2.0)
    O, lse = oracle.attention(q, k, v, mask_kind=mask_kind, window=window, doc_offsets=docs,
                              softcap=30.0)
    Ot, lt = oracle.attention_tiled_online(q, k, v, block_q=bq, block_kv=bk,
                                           mask_kind=mask_kind, window=window,
                                           doc_offsets=docs, softcap=30.0)
    assert np.allclose(O, Ot, atol=1e-12, rtol=0)
    assert np.allclose(lse, lt, atol=1e-12, rtol=0)


@pytest.mark.parametrize("splits,T,tile", [(1, 37, 1), (2, 37, 1), (3, 37, 1), (8, 37, 1),
                                            (37, 37, 1), (3, 200, 64), (5, 200, 64),
                                            (6, 2000, 64)])
def test_split_kv_merge_equals_unsplit(splits, T, tile):
    B, Hq, Hkv, d = 2, 8, 2, 16
    rng = np.random.default_rng(8)
    q = rng.standard_normal((B, Hq, 1, d))
    kc = rng.standard_normal((B, Hkv, T, d))
    vc = rng.standard_normal((B, Hkv, T, d))
    O, lse, _, _ = oracle.decode_splitkv(q, kc, vc, splits, tile=tile)
    Ou, lu = oracle.attention(q, kc, vc)
    assert np.allclose(O, Ou, atol=1e-12, rtol=0)
    assert np.allclose(lse, lu, atol=1e-12, rtol=0)


@pytest.mark.parametrize("T,S,tile", [(37, 8, 1), (2000, 6, 64), (200, 5, 64), (64, 3, 64),
                                      (32768, 15, 64), (1, 4, 64)])
def test_split_bounds_tile_the_keys(T, S, tile):
    b = oracle.split_bounds(T, S, tile)
    assert len(b) == S and b[0][0] == 0 and b[-1][1] == T
    assert all(b[i][1] == b[i + 1][0] for i in range(S - 1))       # contiguous, no overlap
    assert all(t0 <= t1 for t0, t1 in b)
    assert all(t1 % tile == 0 for t0, t1 in b[:-1])                 # cuts only at tile ends
    tiles = [-(-(t1 - t0) // tile) for t0, t1 in b]
    assert max(tiles) - min(tiles) <= 1                             # balanced by whole tiles


def test_merge_with_fully_masked_splits():
    # document mask: the splits outside the query's document have LSE = -inf (weight 0)
    N, d = 20, 8
    q, k, v = _rand_qkv(1, 1, 1, N, d, 9)
    O, lse = oracle.attention(q, k, v, mask_kind=MASK_DOCUMENT_CAUSAL, doc_offsets=DOCS_SMALL)
    rows = np.arange(N)
    parts_o, parts_l = [], []
    for s0, s1 in oracle.split_bounds(N, 5):
        cols = np.arange(s0, s1)
        o, l = oracle.attention_head(q[0, 0], rows, k[0, 0, s0:s1], v[0, 0, s0:s1],
                                     1 / math.sqrt(d), MASK_DOCUMENT_CAUSAL, 0, 0.0,
                                     DOCS_SMALL, kv_idx=cols)
        parts_o.append(o)
        parts_l.append(l)
    assert np.isneginf(np.stack(parts_l, axis=1)).any()
    Om, lm = oracle.merge_partials(np.stack(parts_o, axis=1), np.stack(parts_l, axis=1))
    assert np.allclose(Om, O[0, 0], atol=1e-12, rtol=0)
    assert np.allclose(lm, lse[0, 0], atol=1e-12, rtol=0)


def test_fully_masked_row_gives_zero_and_minus_inf():
    # kv positions beyond the keys of a doc never seen: use a sliding window of -1 so no
    # key is visible at all (window < 0 keeps nothing), the degenerate case of reading c6
    q, k, v = _rand_qkv(1, 1, 1, 4, 8, 10)
    O, lse = oracle.attention(q, k, v, mask_kind=MASK_SLIDING_CAUSAL, window=-1)
    assert np.all(O == 0.0) and np.all(np.isneginf(lse))
    Ot, lt = oracle.attention_tiled_online(q, k, v, mask_kind=MASK_SLIDING_CAUSAL, window=-1)
    assert np.all(Ot == 0.0) and np.all(np.isneginf(lt))


# ------------------------------------------------------------------ tile maps and counts

def _tile_class_by_intervals(i, j, N, bq, bk, mask_kind, window, docs):
    """Classify a tile from each row's visible key interval [lo(q), hi(q)]."""
    q0, q1 = i * bq, min(N, (i + 1) * bq)
    k0, k1 = j * bk, min(N, (j + 1) * bk)
    full, any_ = True, False
    for qq in range(q0, q1):
        if mask_kind == MASK_NONE:
            lo, hi = 0, N - 1
        elif mask_kind == MASK_CAUSAL:
            lo, hi = 0, qq
        elif mask_kind == MASK_SLIDING_CAUSAL:
            lo, hi = max(0, qq - window), qq
        elif mask_kind == MASK_SLIDING:
            lo, hi = max(0, qq - window), min(N - 1, qq + window)
        else:
            lo, hi = max(int(o) for o in docs if o <= qq), qq
        a, b = max(lo, k0), min(hi, k1 - 1)
        if a <= b:
            any_ = True
        if not (lo <= k0 and k1 - 1 <= hi):
            full = False
    return TILE_FULL if full else (TILE_PARTIAL if any_ else TILE_EMPTY)


@pytest.mark.parametrize("mask_kind,window,docs", MASKS)
@pytest.mark.parametrize("bq,bk", [(4, 4), (3, 5), (8, 2)])
def test_tile_map_small_against_intervals(mask_kind, window, docs, bq, bk):
    N = 20
    tm = oracle.tile_map(2, N, N, mask_kind, window, docs, bq, bk)
    for i in range(tm.shape[1]):
        for j in range(tm.shape[2]):
            want = _tile_class_by_intervals(i, j, N, bq, bk, mask_kind, window, docs)
            assert tm[0, i, j] == want and tm[1, i, j] == want


def test_tile_map_causal_4096_counts():
    tm = oracle.tile_map(1, 4096, 4096, MASK_CAUSAL)
    assert (tm == TILE_FULL).sum() == 496 and (tm == TILE_PARTIAL).sum() == 32
    assert np.all(np.diag(tm[0]) == TILE_PARTIAL)


@pytest.mark.slow
def test_tile_map_sliding_16384_w1024_counts():
    # rows i >= 8 of 128-row tiles: 7 full tiles (i-7..i-1) and 2 partial (i-8, i);
    # rows i < 8: i full tiles and the diagonal partial.
    tm = oracle.tile_map(1, 16384, 16384, MASK_SLIDING_CAUSAL, window=1024)
    full = sum(i for i in range(8)) + 120 * 7
    part = 8 + 120 * 2
    assert (tm == TILE_FULL).sum() == full == 868
    assert (tm == TILE_PARTIAL).sum() == part == 248


def test_visible_pair_closed_forms_match_element_counts():
    docs = workloads.doc_offsets_for(3000, 100, 700, seed=3)
    for (kind, w, dd) in [(MASK_NONE, 0, None), (MASK_CAUSAL, 0, None),
                          (MASK_SLIDING_CAUSAL, 257, None), (MASK_SLIDING_CAUSAL, 5000, None),
                          (MASK_DOCUMENT_CAUSAL, 0, docs), (MASK_SLIDING, 0, None),
                          (MASK_SLIDING, 257, None), (MASK_SLIDING, 5000, None)]:
        assert accounting.visible_pairs(3000, 3000, kind, w, dd) == \
            oracle.visible_pairs(3000, 3000, kind, w, dd)
    assert accounting.visible_pairs(16384, 16384, MASK_SLIDING_CAUSAL, 1024) == 16268800


def test_executed_tiles_are_the_non_empty_tiles_of_the_brute_force_map():
    # every key tile a query tile walks holds a visible pair (the row intervals are
    # monotone), so the kernel's executed tiles are exactly the map's non-empty tiles
    docs = workloads.doc_offsets_for(1000, 100, 400, seed=5)
    for (kind, w, dd) in [(MASK_NONE, 0, None), (MASK_CAUSAL, 0, None),
                          (MASK_SLIDING_CAUSAL, 200, None), (MASK_DOCUMENT_CAUSAL, 0, docs),
                          (MASK_SLIDING, 130, None), (MASK_SLIDING, 0, None)]:
        tm = oracle.tile_map(1, 1000, 1000, kind, w, dd)
        assert accounting.executed_tiles(1000, 1000, kind, w, dd) == int((tm != 0).sum()), kind
    assert accounting.executed_tiles(4096, 4096, MASK_CAUSAL) == 528
    assert accounting.executed_tiles(16384, 16384, MASK_SLIDING_CAUSAL, 1024) == 868 + 248


def test_document_generator():
    lens = workloads.doc_lengths(32768, 512, 4096, seed=0)
    assert sum(lens) == 32768 and all(512 <= x <= 4096 for x in lens[:-1])
    assert 1 <= lens[-1] <= 4096
    offs = workloads.doc_offsets_for(32768)
    assert offs[0] == 0 and offs[-1] == 32768 and np.all(np.diff(offs) > 0)
    ids = oracle.document_ids(np.arange(32768), offs)
    assert np.array_equal(np.bincount(ids), np.array(lens))


# ------------------------------------------------------------- byte-accounting closed forms

def test_score_matrix_sizes_printed_on_pages():
    units = {"GB": 1e9, "MiB": 2 ** 20}
    for line in _rows("memory_sizes.txt"):
        _, B, H, N, eb, printed, unit, tol = [x.strip() for x in line.split("|")]
        got = accounting.score_matrix_bytes(int(B), int(H), int(N), int(eb)) / units[unit]
        assert abs(got - float(printed)) <= float(tol) + 5e-3, line
    # FlexAttention page, section 1: 32k tokens -> more than a billion scores per head
    assert 32768 * 32768 > 1e9


def test_gqa_kv_cache_exercise():
    # "3.7 어텐션 II", exercise 3: Hq=32, d=128, fp16, T=16384, B=1; K and V both.
    mib = 2 ** 20
    assert accounting.kv_cache_bytes(32, 16384, 128) == 256 * mib
    assert accounting.kv_cache_bytes(8, 16384, 128) == 64 * mib
    assert accounting.kv_cache_bytes(1, 16384, 128) == 8 * mib
    # the decode workload's KV cache: 8 GiB per step
    w = workloads.DECODE
    assert accounting.decode_kv_bytes(w.B, w.Hkv, w.Nk, w.d) == 8 * 2 ** 30


def test_useful_flops_of_the_prefill_workloads():
    w = workloads.CAUSAL_MHA
    f = accounting.prefill_useful_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.mask_kind)
    assert f == 4 * 128 * (4096 * 4097 // 2) * 8 * 32      # 1.0998 TFLOP
    w = workloads.DOC_SOFTCAP
    docs = workloads.workload_doc_offsets(w)
    pairs = accounting.visible_pairs(w.Nq, w.Nk, w.mask_kind, 0, docs)
    assert pairs == sum(L * (L + 1) // 2 for L in workloads.doc_lengths(32768))


# ------------------------------------------------------------------------ ALiBi bias

def _alibi_weights(i, N, slope, mask_kind):
    """Softmax weights of row i when every raw score is 0: exp(-slope * |i - j|) over the
    visible keys, written out as the geometric sequence it is."""
    js = np.arange(N)
    if mask_kind == MASK_CAUSAL:
        js = js[: i + 1]
    return js, np.exp(-slope * np.abs(i - js).astype(np.float64))


@pytest.mark.parametrize("mask_kind", [MASK_NONE, MASK_CAUSAL])
def test_alibi_equal_scores_closed_form(mask_kind):
    # Q = 0: the scores are the bias alone, so row i weighs key j by exp(-slope |i - j|).
    # Causal: the log-sum-exp is the geometric sum ln((1 - r^(i+1)) / (1 - r)), r = e^-slope.
    N, d = 24, 8
    _, k, v = _rand_qkv(1, 2, 2, N, d, 11)
    q = np.zeros((1, 2, N, d))
    slopes = np.array([0.5, 0.0625])
    O, lse = oracle.attention(q, k, v, mask_kind=mask_kind, alibi_slopes=slopes)
    for h, slope in enumerate(slopes):
        r = math.exp(-slope)
        for i in range(N):
            js, w = _alibi_weights(i, N, slope, mask_kind)
            want = (w[:, None] * v[0, h, js]).sum(axis=0) / w.sum()
            assert np.allclose(O[0, h, i], want, atol=1e-13, rtol=0)
            if mask_kind == MASK_CAUSAL:
                assert abs(lse[0, h, i] - math.log((1 - r ** (i + 1)) / (1 - r))) < 1e-13
            else:
                left = (1 - r ** (i + 1)) / (1 - r)          # j = i, i-1, ..., 0
                right = r * (1 - r ** (N - 1 - i)) / (1 - r)   # j = i+1, ..., N-1
                assert abs(lse[0, h, i] - math.log(left + right)) < 1e-13


def test_alibi_zero_slopes_are_no_bias():
    q, k, v = _rand_qkv(1, 3, 3, 17, 8, 12)
    for kind, w in [(MASK_NONE, 0), (MASK_CAUSAL, 0), (MASK_SLIDING, 4)]:
        O0, l0 = oracle.attention(q, k, v, mask_kind=kind, window=w)
        O1, l1 = oracle.attention(q, k, v, mask_kind=kind, window=w, alibi_slopes=[0, 0, 0])
        assert np.array_equal(O0, O1) and np.array_equal(l0, l1)


@pytest.mark.parametrize("mask_kind,window,docs", MASKS)
def test_alibi_matches_torch_sdpa_float64(mask_kind, window, docs):
    # the bias enters torch's SDPA as an additive float mask (-inf where not visible)
    B, Hq, Hkv, N, d = 2, 4, 2, 19, 16
    q, k, v = _rand_qkv(B, Hq, Hkv, N, d, 13)
    slopes = np.array([1.0, 0.5, 0.25, 0.125])
    scale = 0.2
    O, lse = oracle.attention(q, k, v, scale=scale, mask_kind=mask_kind, window=window,
                              doc_offsets=docs, alibi_slopes=slopes)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    tk = tk.repeat_interleave(Hq // Hkv, dim=1)
    tv = tv.repeat_interleave(Hq // Hkv, dim=1)
    idx = torch.arange(N, dtype=torch.float64)
    dist = (idx[:, None] - idx[None, :]).abs()
    bias = -torch.from_numpy(slopes)[:, None, None] * dist[None]
    bias = bias.masked_fill(~_torch_mask(N, mask_kind, window, docs)[None], float("-inf"))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=bias[None],
                                                           scale=scale)
    assert np.allclose(O, ref.numpy(), atol=1e-8, rtol=0)
    S = torch.einsum("bhid,bhjd->bhij", tq, tk) * scale + bias[None]
    assert np.allclose(lse, torch.logsumexp(S, dim=-1).numpy(), atol=1e-8, rtol=0)


@pytest.mark.parametrize("bq,bk", [(1, 1), (3, 5), (16, 16)])
def test_alibi_tiled_online_equals_full(bq, bk):
    q, k, v = _rand_qkv(1, 2, 1, 21, 8, 14)
    slopes = [0.3, 2.0]
    for kind, w in [(MASK_CAUSAL, 0), (MASK_SLIDING, 5)]:
        O, l = oracle.attention(q, k, v, mask_kind=kind, window=w, alibi_slopes=slopes)
        Ot, lt = oracle.attention_tiled_online(q, k, v, block_q=bq, block_kv=bk, mask_kind=kind,
                                               window=w, alibi_slopes=slopes)
        assert np.allclose(O, Ot, atol=1e-12, rtol=0) and np.allclose(l, lt, atol=1e-12, rtol=0)


# ------------------------------------------------------------- paged, varlen decode

def _paged_case(seed, B=3, Hq=8, Hkv=2, page=4, d=8, lens=(9, 0, 16), max_pages=5):
    rng = np.random.default_rng(seed)
    num_pages = B * max_pages + 2
    kp = rng.standard_normal((num_pages, Hkv, page, d))
    vp = rng.standard_normal((num_pages, Hkv, page, d))
    table = rng.permutation(num_pages)[: B * max_pages].reshape(B, max_pages).astype(np.int32)
    q = rng.standard_normal((B, Hq, 1, d))
    return q, kp, vp, table, np.array(lens, dtype=np.int32)


def test_paged_decode_matches_torch_sdpa_on_gathered_keys():
    q, kp, vp, table, lens = _paged_case(21)
    O, lse = oracle.decode_paged(q, kp, vp, table, lens, scale=0.3)
    B, Hq, _, d = q.shape
    G = Hq // kp.shape[1]
    for b in range(B):
        T = int(lens[b])
        if T == 0:
            assert np.all(O[b] == 0.0) and np.all(np.isneginf(lse[b]))
            continue
        # gather by hand: logical row t lives in page table[b, t // page], slot t % page
        page = kp.shape[2]
        K = torch.stack([torch.from_numpy(kp[table[b, t // page], :, t % page]) for t in range(T)], 1)
        V = torch.stack([torch.from_numpy(vp[table[b, t // page], :, t % page]) for t in range(T)], 1)
        K = K.repeat_interleave(G, dim=0)[None]
        V = V.repeat_interleave(G, dim=0)[None]
        tq = torch.from_numpy(q[b:b + 1])
        ref = torch.nn.functional.scaled_dot_product_attention(tq, K, V, scale=0.3)
        assert np.allclose(O[b:b + 1], ref.numpy(), atol=1e-8, rtol=0)
        S = torch.einsum("bhid,bhjd->bhij", tq, K) * 0.3
        assert np.allclose(lse[b:b + 1], torch.logsumexp(S, -1).numpy(), atol=1e-8, rtol=0)


def test_paged_decode_is_invariant_to_page_placement():
    q, kp, vp, table, lens = _paged_case(22)
    O, lse = oracle.decode_paged(q, kp, vp, table, lens)
    perm = np.random.default_rng(5).permutation(kp.shape[0])     # new slot of each page
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    O2, lse2 = oracle.decode_paged(q, kp2, vp2, perm[table], lens)
    assert np.array_equal(O, O2) and np.array_equal(lse, lse2)


def test_paged_decode_ignores_rows_past_the_length():
    q, kp, vp, table, lens = _paged_case(23, lens=(9, 5, 13))
    O, lse = oracle.decode_paged(q, kp, vp, table, lens)
    kp2, vp2 = kp.copy(), vp.copy()
    page = kp.shape[2]
    for b, T in enumerate(lens):
        last = table[b, (T - 1) // page]
        kp2[last, :, (T - 1) % page + 1:] = 1e6               # the unused tail of the last page
        vp2[last, :, (T - 1) % page + 1:] = -1e6
        for j in range(-(-T // page), table.shape[1]):
            kp2[table[b, j]] = 7.0                           # pages past the length
    O2, lse2 = oracle.decode_paged(q, kp2, vp2, table, lens)
    assert np.array_equal(O, O2) and np.array_equal(lse, lse2)


def test_paged_decode_equal_scores_give_mean_of_the_first_rows():
    q, kp, vp, table, lens = _paged_case(24, lens=(7, 1, 16))
    q = np.zeros_like(q)
    O, lse = oracle.decode_paged(q, kp, vp, table, lens)
    page = kp.shape[2]
    G = q.shape[1] // kp.shape[1]
    for b, T in enumerate(lens):
        rows = np.stack([vp[table[b, t // page], :, t % page] for t in range(T)], 1)   # [Hkv, T, d]
        for h in range(q.shape[1]):
            assert np.allclose(O[b, h, 0], rows[h // G].mean(axis=0), atol=1e-14, rtol=0)
            assert abs(lse[b, h, 0] - math.log(T)) < 1e-14


# ------------------------------------------------------------------------ backward pass

def _fd_grads(q, k, v, W, eps=1e-6, **kw):
    """Central differences of L = sum(O * W) through the forward oracle, element by element."""
    def loss(qq, kk, vv):
        return float((oracle.attention(qq, kk, vv, **kw)[0] * W).sum())
    out = []
    for x in (q, k, v):
        g = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[i] += eps
            xm[i] -= eps
            args_p = [xp if y is x else y for y in (q, k, v)]
            args_m = [xm if y is x else y for y in (q, k, v)]
            g[i] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        out.append(g)
    return out


BWD_CASES = [dict(mask_kind=MASK_NONE), dict(mask_kind=MASK_CAUSAL),
             dict(mask_kind=MASK_SLIDING_CAUSAL, window=2), dict(mask_kind=MASK_SLIDING, window=1),
             dict(mask_kind=MASK_DOCUMENT_CAUSAL, doc_offsets=np.array([0, 2, 3, 6], np.int32)),
             dict(mask_kind=MASK_CAUSAL, softcap=0.7),
             dict(mask_kind=MASK_NONE, alibi_slopes=[0.5, 1.5, 0.25, 0.0])]


@pytest.mark.parametrize("kw", BWD_CASES)
def test_backward_matches_finite_differences(kw):
    # GQA (4 query heads on 2 KV heads), N = 6, d = 3: every gradient element by central
    # differences of the forward oracle
    q, k, v = _rand_qkv(1, 4, 2, 6, 3, 31)
    W = np.random.default_rng(32).standard_normal((1, 4, 6, 3))
    kw = dict(kw, scale=0.7)
    dq, dk, dv = oracle.attention_backward(q, k, v, W, **kw)
    nq, nk, nv = _fd_grads(q, k, v, W, **kw)
    for got, want in ((dq, nq), (dk, nk), (dv, nv)):
        assert np.allclose(got, want, atol=2e-8, rtol=0), np.abs(got - want).max()


@pytest.mark.parametrize("mask_kind,window,docs", MASKS)
def test_backward_matches_torch_autograd_float64(mask_kind, window, docs):
    B, Hq, Hkv, N, d = 2, 4, 2, 19, 8
    q, k, v = _rand_qkv(B, Hq, Hkv, N, d, 33)
    dout = np.random.default_rng(34).standard_normal((B, Hq, N, d))
    scale = 0.3
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, scale=scale, mask_kind=mask_kind,
                                           window=window, doc_offsets=docs)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(G, dim=1), tv.repeat_interleave(G, dim=1),
        attn_mask=_torch_mask(N, mask_kind, window, docs), scale=scale)
    ref.backward(torch.from_numpy(dout))
    for got, want in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.allclose(got, want.numpy(), atol=1e-8, rtol=0)


def test_backward_invariants():
    # each row's dS sums to zero, so shifting every key by one vector leaves dQ unchanged;
    # each visible row's probabilities sum to one, so the dV rows sum to the dO rows' sum
    q, k, v = _rand_qkv(1, 2, 1, 15, 6, 35)
    dout = np.random.default_rng(36).standard_normal((1, 2, 15, 6))
    for kind, w in [(MASK_NONE, 0), (MASK_CAUSAL, 0), (MASK_SLIDING, 3)]:
        dq, dk, dv = oracle.attention_backward(q, k, v, dout, mask_kind=kind, window=w)
        dq2, _, _ = oracle.attention_backward(q, k + np.arange(6.0), v, dout, mask_kind=kind,
                                              window=w)
        assert np.allclose(dq, dq2, atol=1e-12, rtol=0)
        assert np.allclose(dv.sum(axis=2)[0, 0], dout.sum(axis=(1, 2))[0], atol=1e-12, rtol=0)


# ------------------------------------------------------------------------ FP8 inputs

from oracle import fp8 as ofp8  # noqa: E402


@pytest.mark.parametrize("d", [64, 128])
def test_rotation_is_orthogonal_and_keeps_the_scores(d):
    H = ofp8.hadamard(d)
    assert np.array_equal(H @ H.T, d * np.eye(d))
    assert set(np.unique(H)) == {-1.0, 1.0}
    rng = np.random.default_rng(d)
    signs = rng.choice([-1.0, 1.0], size=d)
    q = rng.standard_normal((7, d))
    k = rng.standard_normal((9, d))
    assert np.allclose(ofp8.rotate(q, signs) @ ofp8.rotate(k, signs).T, q @ k.T, atol=1e-12)
    # an outlier column is spread over all columns (incoherence): max |x| drops by sqrt(d)
    x = np.zeros((1, d))
    x[0, 3] = 10.0
    assert np.allclose(np.abs(ofp8.rotate(x, signs)), 10.0 / np.sqrt(d))


@pytest.mark.parametrize("d", [2, 8, 64, 128])
def test_hadamard_entries_and_rotation_of_unit_vectors(d):
    # Sylvester's H has the closed form H[i, j] = (-1)^popcount(i & j); the rotation of the
    # unit vector e_j is row j of H scaled by the j-th sign and 1/sqrt(d)
    H = ofp8.hadamard(d)
    want = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(d)] for i in range(d)])
    assert np.array_equal(H, want)
    signs = np.random.default_rng(d + 1).choice([-1.0, 1.0], size=d)
    R = ofp8.rotate(np.eye(d), signs)
    assert np.allclose(R, signs[:, None] * want / np.sqrt(d), atol=1e-15, rtol=0)


def test_e4m3_grid_points_and_error_bounds():
    # the largest finite E4M3 value is 448; 1 + 2^-3 is a grid point, 1 + 2^-4 a tie that
    # rounds to even (1); normal values round within 2^-4 relative, subnormals (below 2^-6)
    # within half their spacing 2^-9
    vals = ofp8.to_e4m3(np.array([448.0, 1.125, 1.0625, 1.1875, -3.0, 2 ** -9, 2 ** -6]))
    assert list(vals) == [448.0, 1.125, 1.0, 1.25, -3.0, 2 ** -9, 2 ** -6]
    x = np.random.default_rng(3).standard_normal(100000) * 50
    r = ofp8.to_e4m3(x)
    normal = np.abs(x) >= 2 ** -6
    assert np.all(np.abs(r - x)[normal] <= 2 ** -4 * np.abs(x)[normal] + 1e-12)
    assert np.all(np.abs(r - x)[~normal] <= 2 ** -10 + 1e-12)


def test_block_quantization_uses_the_full_range_per_block():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 3, 300, 16)) * np.array([1.0, 100.0, 0.01])[None, :, None, None]
    x[1, 2, 128:256] = 0.0                                   # an all-zero block
    codes, scales = ofp8.quantize_blocks(x, 128)
    assert scales.shape == (2, 3, 3) and scales[1, 2, 1] == 1.0
    assert np.all(codes[1, 2, 128:256] == 0.0)
    for b in range(2):
        for h in range(3):
            for i in range(3):
                blk = codes[b, h, i * 128:(i + 1) * 128]
                if scales[b, h, i] != 1.0 or np.any(blk):
                    assert np.abs(blk).max() == 448.0        # the block's amax maps to 448
    deq = ofp8.dequantize_blocks(codes, scales, 128)
    rep = np.repeat(scales, 128, axis=2)[:, :, :300, None]
    assert np.all(np.abs(deq - x) <= 2 ** -4 * np.abs(x) + rep * 2 ** -10 + 1e-12)


def test_fp8_attention_is_attention_of_the_dequantized_values():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((1, 2, 200, 16)) for _ in range(3))
    qc, qs = ofp8.quantize_blocks(q, 128)
    kc, ks = ofp8.quantize_blocks(k, 128)
    vc, vs = ofp8.quantize_blocks(v, 200)                    # one scale per head
    O, lse = ofp8.attention_fp8(qc, qs, kc, ks, vc, vs[:, :, 0], scale=0.25, mask_kind=1)
    O2, lse2 = oracle.attention(ofp8.dequantize_blocks(qc, qs, 128),
                                ofp8.dequantize_blocks(kc, ks, 128),
                                ofp8.dequantize_blocks(vc, vs, 200), scale=0.25, mask_kind=1)
    assert np.array_equal(O, O2) and np.array_equal(lse, lse2)
    # causal row 0 sees only key 0: O = the dequantized v_0, within E4M3 rounding of v_0
    assert np.all(np.abs(O[0, :, 0] - v[0, :, 0]) <= 2 ** -4 * np.abs(v[0, :, 0])
                  + vs[0, :, 0, None] * 2 ** -10 + 1e-12)
