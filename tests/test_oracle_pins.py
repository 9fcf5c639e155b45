"""Pins for the fp64 CPU oracle: each oracle function is checked against something other than
itself -- hand-derived fixtures (tests/golden), closed forms, library routines (numpy matmul,
torch float64 causal attention), brute-force ranking and invariants of the method (LongCat
Sparse Attention, arXiv 2608.01662).  Chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one test."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from lightning_indexer_top_score_b200.workloads import bf16_bits_to_f32, to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bits(x):
    return to_bf16_bits(np.asarray(x, dtype=np.float32))


def _exact(x):
    """Values already representable in bf16 (the oracle reads bf16 bit patterns)."""
    b = _bits(x)
    assert np.array_equal(bf16_bits_to_f32(b), np.asarray(x, dtype=np.float32))
    return b


# ----------------------------------------------------------------------------- a1 regions

def test_regions_golden():
    g = _golden("regions.json")
    for c in g["cases"]:
        got = oracle.regions(c["t"], c["sink"], c["swa"])
        assert [list(r) for r in got] == c["expect"], c


@pytest.mark.parametrize("Ks,Kw", [(16, 1024), (16, 128), (0, 0), (4, 7), (0, 9), (5, 0)])
def test_regions_partition_prefix(Ks, Kw):
    # the three sets are disjoint and together cover exactly [0, t] (causal prefix)
    for t in list(range(0, 60)) + [1039, 1040, 1041, 5000]:
        (a0, a1), (b0, b1), (c0, c1) = oracle.regions(t, Ks, Kw)
        cover = list(range(a0, a1)) + list(range(b0, b1)) + list(range(c0, c1))
        assert sorted(cover) == list(range(t + 1)), (t, Ks, Kw)
        if t + 1 >= Ks + Kw:
            assert a1 - a0 == Ks and b1 - b0 == Kw
        assert all(s >= Ks for s in range(c0, c1))


# ----------------------------------------------------------------------------- a2 score

def test_score_golden():
    g = _golden("score_example.json")
    q, w = _exact(g["q"]), _exact(g["w"])
    for key, want in zip(g["keys"], g["expect"]):
        assert oracle.score_one(q, w, _exact(key)) == want


def test_score_nonneg_reduces_to_matvec():
    # with q, k >= 0 every dot is >= 0, ReLU is the identity and Eq.1 collapses to
    # (sum_j w_j q_j) . k -- a plain matrix-vector product, heads summed first
    rng = np.random.default_rng(1)
    H, D, L = 7, 32, 50
    q = _bits(np.abs(rng.standard_normal((H, D))))
    w = _bits(rng.standard_normal(H))
    k = _bits(np.abs(rng.standard_normal((L, D))))
    qf, wf, kf = (bf16_bits_to_f32(x).astype(np.float64) for x in (q, w, k))
    want = kf @ (wf @ qf)
    got = oracle.scores(q, w, k, np.arange(L))
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)
    # negating the keys makes every dot <= 0: ReLU zeroes every head
    kneg = _bits(-bf16_bits_to_f32(k))
    assert np.all(oracle.scores(q, w, kneg, np.arange(L)) == 0.0)


def test_score_one_hot_closed_form():
    # q_j = c_j e_{a_j}: q_j . k = c_j k[a_j]  ->  I = sum_j w_j max(0, c_j k[a_j])
    rng = np.random.default_rng(2)
    H, D = 6, 16
    a = rng.integers(0, D, H)
    cj = rng.integers(-3, 4, H).astype(np.float32)
    qv = np.zeros((H, D), np.float32)
    qv[np.arange(H), a] = cj
    wv = rng.integers(-2, 3, H).astype(np.float32)
    for _ in range(20):
        kv = rng.integers(-4, 5, D).astype(np.float32)
        want = sum(wv[j] * max(0.0, cj[j] * kv[a[j]]) for j in range(H))
        assert oracle.score_one(_exact(qv), _exact(wv), _exact(kv)) == want


def test_score_head_pairing():
    # permuting heads jointly (q_j, w_j) leaves I unchanged; permuting w alone does not
    rng = np.random.default_rng(3)
    H, D = 8, 24
    q = _bits(rng.standard_normal((H, D)))
    w = _bits(rng.random(H) * np.arange(1, H + 1))
    k = _bits(rng.standard_normal((40, D)))
    perm = rng.permutation(H)
    base = oracle.scores(q, w, k, np.arange(40))
    np.testing.assert_allclose(oracle.scores(q[perm], w[perm], k, np.arange(40)), base,
                               rtol=1e-13, atol=1e-15)
    assert not np.allclose(oracle.scores(q, w[perm], k, np.arange(40)), base)


# ----------------------------------------------------------------------------- a3 top-K

def _brute_topk(score, pos, K):
    """Rank by counting: element i is selected iff fewer than K others beat it, where j beats
    i when s_j > s_i, or s_j == s_i and p_j < p_i."""
    n = len(score)
    sel = []
    for i in range(n):
        beat = sum(1 for j in range(n) if score[j] > score[i]
                   or (score[j] == score[i] and pos[j] < pos[i]))
        if beat < K:
            sel.append(pos[i])
    sel.sort()
    return sel + [-1] * (K - len(sel))


def test_topk_golden_ties():
    for c in _golden("topk_ties.json")["cases"]:
        got, m = oracle.topk(c["scores"], c["pos"], c["K"])
        assert got.tolist() == c["expect"], c
        assert m == sum(1 for x in c["expect"] if x >= 0)


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force(seed):
    rng = np.random.default_rng(seed)
    for _ in range(25):
        n = int(rng.integers(0, 40))
        K = int(rng.integers(1, 45))
        score = rng.integers(-3, 4, n).astype(np.float64) * 0.5   # many ties
        if seed % 2:
            score = score + rng.standard_normal(n) * 1e-3 * (rng.random(n) < 0.5)
        pos = rng.permutation(1000)[:n]
        got, m = oracle.topk(score, pos, K)
        assert got.tolist() == _brute_topk(score.tolist(), pos.tolist(), K)
        assert m == min(n, K)


def test_topk_whole_domain_and_relabel():
    rng = np.random.default_rng(7)
    score = rng.standard_normal(30)
    pos = np.arange(100, 130)
    got, m = oracle.topk(score, pos, 64)
    assert got[:30].tolist() == list(range(100, 130)) and np.all(got[30:] == -1) and m == 30
    # permuting the candidate order changes nothing (selection is a function of the set)
    perm = rng.permutation(30)
    got2, _ = oracle.topk(score[perm], pos[perm], 10)
    assert got2.tolist() == oracle.topk(score, pos, 10)[0].tolist()


# ----------------------------------------------------------------------------- a4 block means

def test_block_means_closed_form():
    # k[s, d] = s + d/4 (exact in bf16 for s < 64): mean over [nB, min(nB+B, L)) is
    # (lo + hi - 1)/2 + d/4
    L, D, B = 61, 4, 8
    kv = np.array([[s + d / 4.0 for d in range(D)] for s in range(L)], np.float32)
    m = oracle.block_means(_exact(kv), L, B)
    assert m.shape == (8, D)
    for n in range(8):
        lo, hi = n * B, min(n * B + B, L)
        for d in range(D):
            assert m[n, d] == (lo + hi - 1) / 2.0 + d / 4.0


# ----------------------------------------------------------------------------- a5 page score

def _means_bits(k, L, B):
    return to_bf16_bits(oracle.block_means(k, L, B).astype(np.float32))


def test_page_score_singleton_blocks_sum_token_scores():
    # Eq. 9 with sub-block size 1: the mean of a one-token block is the token itself, so the
    # page score is the sum of Eq. 1 over the page's tokens
    rng = np.random.default_rng(4)
    H, D, P, L = 4, 16, 8, 37
    q = _bits(rng.standard_normal((H, D)))
    w = _bits(rng.random(H))
    k = _bits(rng.standard_normal((L, D)))
    km = _means_bits(k, L, 1)
    assert np.array_equal(km, k)
    for p in range((L + P - 1) // P):
        toks = np.arange(p * P, min(p * P + P, L))
        want = oracle.scores(q, w, k, toks).sum()
        assert abs(oracle.page_score(q, w, km, L, P, 1, p) - want) <= 1e-12 * (1 + abs(want))


def test_page_score_one_block_is_score_of_mean_key():
    # sub-block size = page size: one mean per page, Eq. 9 = Eq. 1 on the page-mean key
    rng = np.random.default_rng(5)
    H, D, P, L = 4, 16, 8, 37
    q = _bits(rng.standard_normal((H, D)))
    w = _bits(rng.random(H))
    k = _bits(rng.standard_normal((L, D)))
    km = _means_bits(k, L, P)
    for p in range(km.shape[0]):
        assert oracle.page_score(q, w, km, L, P, P, p) == oracle.score_one(q, w, km[p])


def test_page_score_nonneg_matmul():
    # q, means >= 0: Eq. 9 = (sum_j w_j q_j) . (sum_{n in page} kmean_n)
    rng = np.random.default_rng(6)
    H, D, P, B, L = 5, 8, 16, 4, 45
    q = _bits(np.abs(rng.standard_normal((H, D))))
    w = _bits(rng.random(H))
    k = _bits(np.abs(rng.standard_normal((L, D))))
    km = _means_bits(k, L, B)
    kmf = bf16_bits_to_f32(km).astype(np.float64)
    v = bf16_bits_to_f32(w).astype(np.float64) @ bf16_bits_to_f32(q).astype(np.float64)
    for p in range(3):
        want = v @ kmf[p * (P // B):(p + 1) * (P // B)].sum(0)
        np.testing.assert_allclose(oracle.page_score(q, w, km, L, P, B, p), want, rtol=1e-13)


# ----------------------------------------------------------------------------- f4 MinMax pooling

def _minmax_bits(k, L, B):
    return to_bf16_bits(oracle.block_minmax(k, L, B).astype(np.float32))


def test_block_minmax_golden():
    g = _golden("minmax_pooling.json")
    rows = oracle.block_minmax(_exact(g["keys"]), g["L"], g["B"])
    np.testing.assert_array_equal(rows, np.array(g["rows"]))


def test_block_minmax_is_numpy_reduction():
    # element-wise max / min of each sub-block's present tokens (a partial last block included)
    rng = np.random.default_rng(21)
    L, D, B = 53, 6, 8
    k = _bits(rng.standard_normal((L, D)))
    kf = bf16_bits_to_f32(k).astype(np.float64)
    rows = oracle.block_minmax(k, L, B)
    assert rows.shape == (7, 2 * D)
    for n in range(7):
        blk = kf[n * B:min(L, n * B + B)]
        np.testing.assert_array_equal(rows[n, :D], blk.max(0))
        np.testing.assert_array_equal(rows[n, D:], blk.min(0))


def test_page_score_minmax_golden():
    g = _golden("minmax_pooling.json")
    q, w = _exact(g["q"]), _exact(g["w"])
    kmm = _exact(g["rows"])
    for p, want in enumerate(g["page_scores"]):
        assert oracle.page_score_minmax(q, w, kmm, g["L"], g["P"], g["B"], p) == want


def test_page_score_minmax_singleton_blocks_sum_token_scores():
    # sub-block size 1: k_max = k_min = the token, so the term is q . k and the page score is
    # the sum of Eq. 1 over the page (the size-1 column of Table 11, equal for both poolings)
    rng = np.random.default_rng(22)
    H, D, P, L = 4, 16, 8, 37
    q = _bits(rng.standard_normal((H, D)))
    w = _bits(rng.random(H))
    k = _bits(rng.standard_normal((L, D)))
    kmm = _minmax_bits(k, L, 1)
    assert np.array_equal(kmm[:, :D], k) and np.array_equal(kmm[:, D:], k)
    for p in range((L + P - 1) // P):
        toks = np.arange(p * P, min(p * P + P, L))
        want = oracle.scores(q, w, k, toks).sum()
        got = oracle.page_score_minmax(q, w, kmm, L, P, 1, p)
        assert abs(got - want) <= 1e-12 * (1 + abs(want))


def test_page_score_minmax_bounds_every_token_and_the_mean():
    # the term is the largest q . x over the box [k_min, k_max], which holds every token of the
    # sub-block and its mean; with w >= 0 the page score is therefore at least the sum over
    # sub-blocks of their best token's Eq. 1 score, and at least the mean-pooled Eq. 9 score
    rng = np.random.default_rng(23)
    H, D, P, B, L = 4, 16, 32, 8, 200
    q = _bits(rng.standard_normal((H, D)))
    w = _bits(rng.random(H))
    k = _bits(rng.standard_normal((L, D)))
    kmm, km = _minmax_bits(k, L, B), _means_bits(k, L, B)
    tok = oracle.scores(q, w, k, np.arange(L))
    for p in range((L + P - 1) // P):
        got = oracle.page_score_minmax(q, w, kmm, L, P, B, p)
        best = sum(tok[n * B:min(L, n * B + B)].max()
                   for n in range(p * P // B, min((L + B - 1) // B, (p + 1) * P // B)))
        assert got >= best - 1e-12 * (1 + abs(best))
        assert got >= oracle.page_score(q, w, km, L, P, B, p) - 1e-9


def test_page_score_minmax_sign_closed_forms():
    # q >= 0 and keys >= 0: every term picks k_max and is >= 0, so the page score is
    # (sum_j w_j q_j) . (sum_n k_max_n); q <= 0 and keys <= 0: every term picks k_min
    rng = np.random.default_rng(24)
    H, D, P, B, L = 5, 8, 16, 4, 45
    w = _bits(rng.random(H))
    wf = bf16_bits_to_f32(w).astype(np.float64)
    for sign in (1.0, -1.0):
        q = _bits(sign * np.abs(rng.standard_normal((H, D))))
        k = _bits(sign * np.abs(rng.standard_normal((L, D))))
        kmm = _minmax_bits(k, L, B)
        kf = bf16_bits_to_f32(kmm).astype(np.float64)
        v = wf @ bf16_bits_to_f32(q).astype(np.float64)
        half = slice(0, D) if sign > 0 else slice(D, 2 * D)
        for p in range(3):
            want = v @ kf[p * (P // B):(p + 1) * (P // B), half].sum(0)
            np.testing.assert_allclose(oracle.page_score_minmax(q, w, kmm, L, P, B, p), want,
                                       rtol=1e-13)


@pytest.mark.parametrize("B", [1, 8])
def test_index_hi_minmax_equals_flat_when_all_pages_recalled(B):
    q, w, k = _setup_idx(25, L=1000)
    kmm = _minmax_bits(k, 1000, B)
    for t in (999, 700, 300):
        flat, _ = oracle.index_query(q, w, k, None, 1000, t, 50, 16, 64)
        hi, _ = oracle.index_query(q, w, k, kmm, 1000, t, 50, 16, 64, page=32, sub_block=B,
                                   M=1000 // 32 + 1, pooling="minmax")
        assert hi.tolist() == flat.tolist()


def test_index_hi_minmax_restricts_to_top_pages():
    P, B, M, L, t, Ks, Kw, K = 32, 8, 5, 1000, 999, 16, 64, 40
    q, w, k = _setup_idx(26, L=L)
    kmm = _minmax_bits(k, L, B)
    (_, _), (_, _), (lo, hi) = oracle.regions(t, Ks, Kw)
    pages = np.arange(lo // P, (hi - 1) // P + 1)
    ps = np.array([oracle.page_score_minmax(q, w, kmm, L, P, B, p) for p in pages])
    top = sorted(_brute_topk(ps.tolist(), pages.tolist(), M))
    dom = np.array([s for p in top if p >= 0 for s in range(p * P, p * P + P) if lo <= s < hi])
    want = _brute_topk(oracle.scores(q, w, k, dom).tolist(), dom.tolist(), K)
    got, _ = oracle.index_query(q, w, k, kmm, L, t, K, Ks, Kw, page=P, sub_block=B, M=M,
                                pooling="minmax")
    assert got.tolist() == want
    # the batched entry point agrees
    kv = np.array([L], np.int32)
    b = oracle.index(q[None, None], w[None, None], k[None], kmm[None], kv,
                     np.array([[t]], np.int32), K, Ks, Kw, P, B, M, pooling="minmax")
    assert b[0, 0].tolist() == want


# ----------------------------------------------------------------------------- a6 indexer

def _setup_idx(seed, L=700, H=4, D=16):
    rng = np.random.default_rng(seed)
    q = _bits(rng.standard_normal((H, D)) / 4)
    w = _bits(rng.random(H))
    k = _bits(rng.standard_normal((L, D)) / 4)
    return q, w, k


@pytest.mark.parametrize("t,Ks,Kw,K", [(699, 16, 64, 40), (699, 0, 0, 80), (80, 16, 64, 40),
                                       (90, 16, 64, 40), (699, 16, 64, 5000)])
def test_index_flat_is_brute_topk_over_dyn(t, Ks, Kw, K):
    q, w, k = _setup_idx(8)
    (_, _), (_, _), (lo, hi) = oracle.regions(t, Ks, Kw)
    dom = np.arange(lo, hi)
    sc = oracle.scores(q, w, k, dom)
    got, m = oracle.index_query(q, w, k, None, 700, t, K, Ks, Kw)
    assert got.tolist() == _brute_topk(sc.tolist(), dom.tolist(), K)
    assert m == min(K, hi - lo)


@pytest.mark.parametrize("B", [1, 4, 8])
def test_index_hi_equals_flat_when_all_pages_recalled(B):
    q, w, k = _setup_idx(9, L=1000)
    km = _means_bits(k, 1000, B)
    for t in (999, 700, 300):
        flat, _ = oracle.index_query(q, w, k, None, 1000, t, 50, 16, 64)
        hi, _ = oracle.index_query(q, w, k, km, 1000, t, 50, 16, 64, page=32, sub_block=B,
                                   M=1000 // 32 + 1)
        assert hi.tolist() == flat.tolist()


def test_index_hi_restricts_to_top_pages():
    P, B, M, L, t, Ks, Kw, K = 32, 8, 5, 1000, 999, 16, 64, 40
    q, w, k = _setup_idx(10, L=L)
    km = _means_bits(k, L, B)
    (_, _), (_, _), (lo, hi) = oracle.regions(t, Ks, Kw)
    pages = np.arange(lo // P, (hi - 1) // P + 1)
    ps = np.array([oracle.page_score(q, w, km, L, P, B, p) for p in pages])
    # brute-force page ranking, ties to lower page id
    top = sorted(_brute_topk(ps.tolist(), pages.tolist(), M))
    dom = np.array([s for p in top if p >= 0 for s in range(p * P, p * P + P) if lo <= s < hi])
    want = _brute_topk(oracle.scores(q, w, k, dom).tolist(), dom.tolist(), K)
    got, _ = oracle.index_query(q, w, k, km, L, t, K, Ks, Kw, page=P, sub_block=B, M=M)
    assert got.tolist() == want
    assert set(s // P for s in got if s >= 0) <= set(top)


def test_select_from_scores_matches_index():
    # the selection-only entry point, fed the oracle's own scores, reproduces the indexer
    P, B, L, t = 32, 8, 1000, 999
    q, w, k = _setup_idx(11, L=L)
    km = _means_bits(k, L, B)
    tok = oracle.scores(q, w, k, np.arange(L)).astype(np.float32)
    pg = np.array([oracle.page_score(q, w, km, L, P, B, p) for p in range(L // P + 1)],
                  np.float32)
    for M in (0, 4):
        a, _ = oracle.select_query(tok, pg, t, 40, 16, 64, page=P, M=M)
        # recompute with float32-rounded scores through the brute-force ranker
        (_, _), (_, _), (lo, hi) = oracle.regions(t, 16, 64)
        if M == 0:
            dom = np.arange(lo, hi)
        else:
            pages = np.arange(lo // P, (hi - 1) // P + 1)
            top = [p for p in _brute_topk(pg[pages].astype(np.float64).tolist(),
                                          pages.tolist(), M) if p >= 0]
            dom = np.array([s for p in top for s in range(p * P, p * P + P) if lo <= s < hi])
        assert a.tolist() == _brute_topk(tok[dom].astype(np.float64).tolist(), dom.tolist(), 40)


def test_index_batched_matches_per_query():
    rng = np.random.default_rng(12)
    Bn, T, H, D, Lmax = 2, 3, 4, 16, 300
    q = _bits(rng.standard_normal((Bn, T, H, D)))
    w = _bits(rng.random((Bn, T, H)))
    k = _bits(rng.standard_normal((Bn, Lmax, D)))
    kv_len = np.array([300, 250], np.int32)
    q_pos = np.array([[299, 200, 100], [249, 248, 150]], np.int32)
    km = np.stack([_means_bits(k[b], Lmax, 8) for b in range(Bn)])
    for M in (0, 3):
        out = oracle.index(q, w, k, km, kv_len, q_pos, 20, 4, 16, page=32, sub_block=8, M=M)
        for b in range(Bn):
            for i in range(T):
                want, _ = oracle.index_query(q[b, i], w[b, i], k[b], km[b], kv_len[b],
                                             q_pos[b, i], 20, 4, 16, page=32, sub_block=8, M=M)
                assert out[b, i].tolist() == want.tolist()


# ----------------------------------------------------------------------------- a7 attention

def test_attention_golden_two_keys():
    g = _golden("attention_two_keys.json")
    q = _exact([g["q"]])
    c = _exact(g["c"])
    out, lse = oracle.attend_query(q, c, np.array([-1], np.int32), 1, 1, 1, 2, g["scale"])
    np.testing.assert_allclose(out[0], g["expect_out"], rtol=1e-14)
    assert abs(lse[0] - g["expect_lse"]) < 1e-14


def test_attention_uniform_keys_closed_form():
    # identical rows: softmax is uniform over |S_t|, out = v, lse = z + log|S_t|
    rng = np.random.default_rng(13)
    H, Dqk, Dv, L = 3, 24, 16, 300
    row = _bits(rng.standard_normal(Dqk))
    c = np.tile(row, (L, 1))
    q = _bits(rng.standard_normal((H, Dqk)))
    idx = np.array([20, 45, 99, 150, -1, -1], np.int32)
    t, Ks, Kw, scale = 299, 4, 64, 0.3
    out, lse = oracle.attend_query(q, c, idx, t, Ks, Kw, Dv, scale)
    n = Ks + Kw + 4
    rf = bf16_bits_to_f32(row).astype(np.float64)
    for h in range(H):
        z = scale * float(bf16_bits_to_f32(q[h]).astype(np.float64) @ rf)
        np.testing.assert_allclose(out[h], rf[:Dv], rtol=1e-13)
        assert abs(lse[h] - (z + math.log(n))) < 1e-12


def test_attention_dense_causal_matches_torch_sdpa():
    # with every dynamic position selected, the LSA attention of each query is textbook causal
    # softmax attention over 0..t (library routine, float64)
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(14)
    H, Dqk, Dv, L = 4, 40, 32, 96
    scale = 1.0 / math.sqrt(Dqk)
    c = _bits(rng.standard_normal((L, Dqk)))
    qs = _bits(rng.standard_normal((L, H, Dqk)))
    cf = torch.from_numpy(bf16_bits_to_f32(c).astype(np.float64))
    qf = torch.from_numpy(bf16_bits_to_f32(qs).astype(np.float64)).permute(1, 0, 2)  # [H,L,D]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qf, cf.expand(H, L, Dqk), cf[:, :Dv].expand(H, L, Dv), is_causal=True, scale=scale)
    for Ks, Kw in ((0, 0), (3, 10)):
        for t in (0, 5, 13, 50, 95):
            (_, _), (_, _), (lo, hi) = oracle.regions(t, Ks, Kw)
            idx = np.full(L, -1, np.int32)
            idx[:hi - lo] = np.arange(lo, hi)
            out, _ = oracle.attend_query(qs[t], c, idx, t, Ks, Kw, Dv, scale)
            np.testing.assert_allclose(out, ref[:, t].numpy(), rtol=1e-11, atol=1e-12)


def test_attention_branch_merge_equals_single_softmax():
    # Sec. 4.1.1: contiguous and sparse branches merged by LSE rescaling = one softmax over
    # the disjoint union
    rng = np.random.default_rng(15)
    H, Dqk, Dv, L = 4, 32, 24, 500
    c = _bits(rng.standard_normal((L, Dqk)))
    q = _bits(rng.standard_normal((H, Dqk)))
    for t, Ks, Kw, nidx in ((499, 16, 64, 30), (499, 0, 0, 50), (70, 16, 64, 0), (10, 16, 64, 0)):
        (_, _), (_, _), (lo, hi) = oracle.regions(t, Ks, Kw)
        idx = np.full(max(nidx, 1), -1, np.int32)
        if hi > lo and nidx:
            sel = np.sort(rng.choice(np.arange(lo, hi), size=min(nidx, hi - lo), replace=False))
            idx[:len(sel)] = sel
        o1, l1 = oracle.attend_query(q, c, idx, t, Ks, Kw, Dv, 0.2)
        o2, l2 = oracle.attend_query(q, c, idx, t, Ks, Kw, Dv, 0.2, branches=True)
        np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(l2, l1, rtol=1e-12, atol=1e-12)
        # order of the index list is irrelevant
        o3, _ = oracle.attend_query(q, c, idx[::-1].copy(), t, Ks, Kw, Dv, 0.2)
        np.testing.assert_allclose(o3, o1, rtol=1e-12, atol=1e-12)


def test_attention_batched_matches_per_query_and_cli_reuse():
    # batched call = per-query call; a Cross-Layer-Indexing reuse layer (Sec. 3.2) is the same
    # call with the owner's index array, which the call leaves untouched
    rng = np.random.default_rng(16)
    Bn, T, H, Dqk, Dv, L, K = 2, 2, 3, 20, 16, 200, 12
    q = _bits(rng.standard_normal((Bn, T, H, Dqk)))
    c = _bits(rng.standard_normal((Bn, L, Dqk)))
    q_pos = np.array([[199, 150], [120, 199]], np.int32)
    idx = np.full((Bn, T, K), -1, np.int32)
    for b in range(Bn):
        for i in range(T):
            (_, _), (_, _), (lo, hi) = oracle.regions(q_pos[b, i], 4, 32)
            idx[b, i, :8] = np.sort(rng.choice(np.arange(lo, hi), 8, replace=False))
    before = idx.copy()
    out, lse = oracle.attend(q, c, idx, q_pos, 4, 32, Dv, 0.25)
    assert np.array_equal(idx, before)
    for b in range(Bn):
        for i in range(T):
            o, l = oracle.attend_query(q[b, i], c[b], idx[b, i], q_pos[b, i], 4, 32, Dv, 0.25)
            np.testing.assert_array_equal(out[b, i], o)
            np.testing.assert_array_equal(lse[b, i], l)


# ----------------------------------------------------------------------------- planted mistakes

def test_pins_catch_planted_mistakes():
    """Each pin above must reject a plausible mistake.  Plant mistakes in copies of the oracle's
    own C source (CPU only), rebuild, and check that a pin fails."""
    import ctypes
    import subprocess
    import tempfile
    src = open(os.path.join(os.path.dirname(oracle.__file__), "lsa_oracle.c")).read()
    mutations = {
        "relu dropped": ("if (dot > 0.0) I += bf(w[j]) * dot;", "I += bf(w[j]) * dot;"),
        "tie toward higher position": ("return (x->p < y->p) ? -1 : (x->p > y->p);",
                                       "return (x->p > y->p) ? -1 : (x->p < y->p);"),
        "swa off by one": ("int64_t swa_lo = t - Kw + 1;", "int64_t swa_lo = t - Kw;"),
        "minmax extremes swapped": ("double a = qd * bf(kmm_seq[n * 2 * D + d]);      /* q * k_max */",
                                    "double a = qd * bf(kmm_seq[n * 2 * D + D + d]);  /* q * k_max */"),
        "minmax takes the smaller product": ("st += a > b ? a : b;", "st += a < b ? a : b;"),
    }
    golden_score = _golden("score_example.json")
    for name, (a, b) in mutations.items():
        assert a in src, name
        with tempfile.TemporaryDirectory() as d:
            cpath, sopath = os.path.join(d, "m.c"), os.path.join(d, "m.so")
            open(cpath, "w").write(src.replace(a, b))
            subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-fopenmp", cpath, "-o", sopath,
                            "-lm"], check=True)
            lib = ctypes.CDLL(sopath)
            P = ctypes.c_void_p
            if name == "relu dropped":
                lib.orc_score_one.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int]
                lib.orc_score_one.restype = ctypes.c_double
                q, w = _exact(golden_score["q"]), _exact(golden_score["w"])
                k0 = _exact(golden_score["keys"][0])
                got = lib.orc_score_one(q.ctypes.data_as(P), w.ctypes.data_as(P),
                                        k0.ctypes.data_as(P), 2, 2)
                assert got != golden_score["expect"][0]
            elif name == "tie toward higher position":
                lib.orc_topk.argtypes = [P, P, ctypes.c_int64, ctypes.c_int, P]
                lib.orc_topk.restype = ctypes.c_int64
                s = np.zeros(5)
                p = np.arange(10, 15, dtype=np.int64)
                out = np.zeros(3, np.int32)
                lib.orc_topk(s.ctypes.data_as(P), p.ctypes.data_as(P), 5, 3, out.ctypes.data_as(P))
                assert out.tolist() != [10, 11, 12]
            elif name.startswith("minmax"):
                g = _golden("minmax_pooling.json")
                lib.orc_page_score_minmax.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_int64]
                lib.orc_page_score_minmax.restype = ctypes.c_double
                q, w, kmm = _exact(g["q"]), _exact(g["w"]), _exact(g["rows"])
                got = [lib.orc_page_score_minmax(q.ctypes.data_as(P), w.ctypes.data_as(P),
                                                 kmm.ctypes.data_as(P), 2, 2, g["L"], g["P"],
                                                 g["B"], p) for p in range(2)]
                assert got != g["page_scores"], name
            else:
                lib.orc_regions.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, P]
                r = np.zeros(6, np.int64)
                lib.orc_regions(131071, 16, 1024, r.ctypes.data_as(P))
                assert r.tolist() != [0, 16, 130048, 131072, 16, 130048]


# ----------------------------------------------------------------------------- FP8 indexer

def test_e4m3_codes_match_the_format_definition():
    g = _golden("e4m3.json")
    for c in g["decode"]:
        assert oracle.e4m3_value(c["code"]) == c["value"], c
    for c in g["encode"]:
        assert oracle.e4m3_encode(c["y"]) == c["code"], c


def test_e4m3_encode_matches_torch_float8_in_range():
    """torch's float8_e4m3fn cast (round to nearest even) as an independent implementation, on
    random fp32 values inside the finite range, including exact midpoints."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    ys = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.uniform(-3, 2, 3000),
                         [oracle.e4m3_value(c) * 1.0 for c in range(1, 126)]]).astype(np.float32)
    # midpoints between neighbouring codes (exact in fp32)
    mids = np.array([(oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2 for c in range(0, 125)],
                    dtype=np.float32)
    ys = np.concatenate([ys, mids, -mids])
    ys = ys[np.abs(ys) < 448.0]
    ref = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(y)) for y in ys], dtype=np.uint8)
    # -0.0 and +0.0 both decode to 0; compare values, then codes away from zero
    np.testing.assert_array_equal([oracle.e4m3_value(c) for c in got],
                                  [oracle.e4m3_value(c) for c in ref])


def test_e4m3_roundtrip_error_bound():
    """|decode(encode(y)) - y| is at most half a step: 2^-4 |y| for normal values, 2^-10 below."""
    rng = np.random.default_rng(1)
    ys = (rng.standard_normal(5000) * 10.0 ** rng.uniform(-4, 2.5, 5000)).astype(np.float32)
    ys = ys[np.abs(ys) <= 448.0]
    for y in ys:
        v = oracle.e4m3_value(oracle.e4m3_encode(float(y)))
        bound = 2.0 ** -4 * abs(float(y)) if abs(y) >= 2.0 ** -6 else 2.0 ** -10
        assert abs(v - float(y)) <= bound + 1e-30, (y, v)


def test_quantize_rows():
    """Per-row scale amax / 448: the largest element of a row maps to +-448 exactly, every code
    decodes to within half a step of x / scale, and an all-zero row has scale 0 and zero codes."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((6, 128)).astype(np.float32) * np.array([1e-3, 0.1, 1, 3, 100, 1e4],
                                                                       np.float32)[:, None]
    x[5] = 0.0
    xb = to_bf16_bits(x)
    codes, scales = oracle.quantize_e4m3(xb)
    xf = bf16_bits_to_f32(xb)
    for r in range(5):
        amax = np.abs(xf[r]).max()
        assert scales[r] == np.float32(amax) / np.float32(448.0)
        j = int(np.abs(xf[r]).argmax())
        assert abs(oracle.e4m3_value(codes[r, j])) == 448.0
        y = xf[r] / scales[r]
        v = np.array([oracle.e4m3_value(c) for c in codes[r]])
        assert np.all(np.abs(v - y) <= np.maximum(2.0 ** -4 * np.abs(y), 2.0 ** -10) + 1e-6)
    assert scales[5] == 0.0 and not codes[5].any()


def test_fp8_score_reduces_to_eq1_on_representable_rows():
    """When every element is an E4M3 value and each row's largest magnitude is 448, the scales
    are 1 and the codes are exact, so the FP8 score equals Eq. 1 (the bf16 oracle) on the same
    values -- and scaling a key row by 2^k scales its score by 2^k (ReLU is homogeneous)."""
    rng = np.random.default_rng(3)
    H, D, n = 8, 64, 20
    pool = np.array([oracle.e4m3_value(c) for c in range(0, 127)] +
                    [-oracle.e4m3_value(c) for c in range(1, 127)], np.float32)
    q = rng.choice(pool, (H, D)).astype(np.float32)
    k = rng.choice(pool, (n, D)).astype(np.float32)
    q[:, 0] = 448.0
    k[:, 0] = -448.0
    w = to_bf16_bits(rng.uniform(0.1, 1.0, H).astype(np.float32))
    qb, kb = to_bf16_bits(q), to_bf16_bits(k)  # E4M3 values are exact in bf16
    q8, qs = oracle.quantize_e4m3(qb)
    k8, ks = oracle.quantize_e4m3(kb)
    assert np.all(qs == 1.0) and np.all(ks == 1.0)
    pos = np.arange(n)
    np.testing.assert_array_equal(oracle.scores_fp8(q8, qs, w, k8, ks, pos),
                                  oracle.scores(qb, w, kb, pos))
    ks2 = ks * np.float32(4.0)
    np.testing.assert_array_equal(oracle.scores_fp8(q8, qs, w, k8, ks2, pos),
                                  4.0 * oracle.scores(qb, w, kb, pos))


def test_fp8_pins_catch_planted_rounding_mistake():
    """A ties-away encoder (a plausible slip) is rejected by the tie fixture."""
    import ctypes
    import subprocess
    import tempfile
    src = open(os.path.join(os.path.dirname(oracle.__file__), "lsa_oracle.c")).read()
    a = "if (d < best_d || (d == best_d && (c & 1) == 0)) {"
    assert a in src
    with tempfile.TemporaryDirectory() as d:
        cpath, sopath = os.path.join(d, "m.c"), os.path.join(d, "m.so")
        open(cpath, "w").write(src.replace(a, "if (d <= best_d) {"))
        subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-fopenmp", cpath, "-o", sopath, "-lm"],
                       check=True)
        lib = ctypes.CDLL(sopath)
        lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        got = [lib.orc_e4m3_encode(c["y"]) for c in _golden("e4m3.json")["encode"]]
        assert got != [c["code"] for c in _golden("e4m3.json")["encode"]]


# ----------------------------------------------------------------------------- HFA backward

def _torch_attention_grads(qf, cf, q_pos, Dv, scale, dout):
    """Dense causal attention in torch float64 with autograd: query i of one sequence attends
    keys 0..q_pos[i]; returns (dq [T,H,Dqk], dc [L,Dqk]) of sum(out * dout)."""
    torch = pytest.importorskip("torch")
    q = torch.tensor(qf, dtype=torch.float64, requires_grad=True)
    c = torch.tensor(cf, dtype=torch.float64, requires_grad=True)
    T, L = q.shape[0], c.shape[0]
    z = scale * torch.einsum("thd,ld->thl", q, c)
    mask = torch.arange(L)[None, :] <= torch.as_tensor(q_pos)[:, None]
    z = z.masked_fill(~mask[:, None, :], float("-inf"))
    out = torch.einsum("thl,ld->thd", torch.softmax(z, dim=-1), c[:, :Dv])
    (out * torch.tensor(dout)).sum().backward()
    return q.grad.numpy(), c.grad.numpy()


def test_attend_bwd_equals_torch_autograd():
    """DSA-mode rows (every position 0..t selected) are plain causal attention: the oracle's
    gradients equal torch float64 autograd, including rows shared by several queries."""
    rng = np.random.default_rng(11)
    L, T, H, Dqk, Dv = 40, 5, 3, 24, 16
    c = to_bf16_bits(rng.standard_normal((L, Dqk)).astype(np.float32))
    q = to_bf16_bits(rng.standard_normal((T, H, Dqk)).astype(np.float32))
    q_pos = np.array([39, 20, 7, 0, 33], np.int32)
    dout = rng.standard_normal((T, H, Dv))
    scale = 0.3
    K = L
    idx = np.full((T, K), -1, np.int32)
    for i, t in enumerate(q_pos):
        idx[i, :t + 1] = np.arange(t + 1)
    dq, dc = oracle.attend_bwd(q[None], c[None], idx[None], q_pos[None], 0, 0, Dv, scale,
                               dout[None])
    tq, tc = _torch_attention_grads(bf16_bits_to_f32(q).astype(np.float64),
                                    bf16_bits_to_f32(c).astype(np.float64), q_pos, Dv, scale, dout)
    np.testing.assert_allclose(dq[0], tq, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dc[0], tc, rtol=1e-10, atol=1e-12)


def test_attend_bwd_streaming_set_equals_torch_on_that_set():
    """With sink, window and sparse picks, the gradients equal those of attention over exactly
    S_t (torch on the gathered rows), and rows outside every S_t get zero gradient."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(12)
    L, H, Dqk, Dv = 64, 2, 16, 8
    c = to_bf16_bits(rng.standard_normal((L, Dqk)).astype(np.float32))
    q = to_bf16_bits(rng.standard_normal((H, Dqk)).astype(np.float32))
    t, sink, swa = 60, 4, 8
    idx = np.array([9, 20, 31, 40, -1, -1], np.int32)
    dout = rng.standard_normal((H, Dv))
    dq, dc = oracle.attend_bwd_query(q, c, idx, t, sink, swa, Dv, 0.5, dout)
    S = np.concatenate([np.arange(0, 4), np.arange(53, 61), idx[idx >= 0]])
    cs = bf16_bits_to_f32(c)[S].astype(np.float64)
    qt = torch.tensor(bf16_bits_to_f32(q).astype(np.float64), requires_grad=True)
    ct = torch.tensor(cs, requires_grad=True)
    p = torch.softmax(0.5 * qt @ ct.T, dim=-1)
    ((p @ ct[:, :Dv]) * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dc[S], ct.grad.numpy(), rtol=1e-10, atol=1e-12)
    outside = np.setdiff1d(np.arange(L), S)
    assert not dc[outside].any()


def test_attend_bwd_single_key_closed_form():
    """One key: p = 1, so dz = 0, dq = 0, and the row's gradient is dout on its first Dv dims."""
    rng = np.random.default_rng(13)
    H, Dqk, Dv = 2, 8, 4
    c = to_bf16_bits(rng.standard_normal((1, Dqk)).astype(np.float32))
    q = to_bf16_bits(rng.standard_normal((H, Dqk)).astype(np.float32))
    dout = rng.standard_normal((H, Dv))
    dq, dc = oracle.attend_bwd_query(q, c, np.array([-1], np.int32), 0, 1, 0, Dv, 0.7, dout)
    assert not dq.any()
    np.testing.assert_allclose(dc[0, :Dv], dout.sum(axis=0), rtol=1e-15)
    assert not dc[0, Dv:].any()


def test_attend_bwd_two_key_closed_form():
    """Two keys: with p the softmax of the two logits, the softmax Jacobian collapses to p1 p2, so
    per head dq = scale p1 p2 (dp1 - dp2) (c1 - c2), and the rows get
    +-scale p1 p2 (dp1 - dp2) q + p_s dout (the second term on the value dims)."""
    rng = np.random.default_rng(14)
    H, Dqk, Dv, scale = 3, 8, 4, 0.6
    c = to_bf16_bits(rng.standard_normal((2, Dqk)).astype(np.float32))
    q = to_bf16_bits(rng.standard_normal((H, Dqk)).astype(np.float32))
    dout = rng.standard_normal((H, Dv))
    # t = 1 with one sink and no window: S_t = {0, 1}
    dq, dc = oracle.attend_bwd_query(q, c, np.array([1], np.int32), 1, 1, 0, Dv, scale, dout)
    cf = bf16_bits_to_f32(c).astype(np.float64)
    qf = bf16_bits_to_f32(q).astype(np.float64)
    want_dq = np.zeros((H, Dqk))
    want_dc = np.zeros((2, Dqk))
    for h in range(H):
        z1, z2 = scale * qf[h] @ cf[0], scale * qf[h] @ cf[1]
        p1 = 1.0 / (1.0 + np.exp(z2 - z1))
        p2 = 1.0 - p1
        g = p1 * p2 * (dout[h] @ cf[0, :Dv] - dout[h] @ cf[1, :Dv])
        want_dq[h] = scale * g * (cf[0] - cf[1])
        want_dc[0] += scale * g * qf[h]
        want_dc[1] -= scale * g * qf[h]
        want_dc[0, :Dv] += p1 * dout[h]
        want_dc[1, :Dv] += p2 * dout[h]
    np.testing.assert_allclose(dq, want_dq, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dc[:2], want_dc, rtol=1e-12, atol=1e-14)


def test_attend_bwd_pin_catches_dropped_term():
    """Dropping the D term of dz (a plausible slip) is rejected by the autograd comparison."""
    import ctypes
    import subprocess
    import tempfile
    src = open(os.path.join(os.path.dirname(oracle.__file__), "lsa_oracle.c")).read()
    a = "const double dz = p * (dp[i] - D);"
    assert a in src
    rng = np.random.default_rng(14)
    L, H, Dqk, Dv = 12, 2, 8, 4
    c = to_bf16_bits(rng.standard_normal((L, Dqk)).astype(np.float32))
    q = to_bf16_bits(rng.standard_normal((H, Dqk)).astype(np.float32))
    dout = rng.standard_normal((H, Dv))
    tq, _ = _torch_attention_grads(bf16_bits_to_f32(q[None]).astype(np.float64),
                                   bf16_bits_to_f32(c).astype(np.float64), np.array([11]), Dv, 0.5,
                                   dout[None])
    with tempfile.TemporaryDirectory() as d:
        cpath, sopath = os.path.join(d, "m.c"), os.path.join(d, "m.so")
        open(cpath, "w").write(src.replace(a, "const double dz = p * dp[i];"))
        subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-fopenmp", cpath, "-o", sopath, "-lm"],
                       check=True)
        lib = ctypes.CDLL(sopath)
        P = ctypes.c_void_p
        lib.orc_attend_bwd_query.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_double, P, P, P]
        idx = np.arange(L, dtype=np.int32)
        dq = np.zeros((H, Dqk))
        dc = np.zeros((L, Dqk))
        lib.orc_attend_bwd_query(q.ctypes.data_as(P), c.ctypes.data_as(P), idx.ctypes.data_as(P),
                                 L, 11, 0, 0, H, Dqk, Dv, 0.5, dout.ctypes.data_as(P),
                                 dq.ctypes.data_as(P), dc.ctypes.data_as(P))
        assert not np.allclose(dq, tq[0], rtol=1e-6)
