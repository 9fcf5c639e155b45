"""Parity of the CUDA path (through the C-ABI) with the fp64 CPU oracle, element by element, on
seeded inputs sized so the oracle answers in seconds while the kernels still cross several tiles
and a ragged tail.  Scores within the stated tolerance; index sets bit-exact when the oracle
selects from the GPU's own scores; attention within bf16 tolerance."""
import numpy as np
import pytest

import oracle
from lightning_indexer_top_score_b200 import lsa
from lightning_indexer_top_score_b200.workloads import (TINY, LsaConfig, bf16_bits_to_f32,
                                                        make_host_inputs, to_bf16_bits)
from _hi_checks import check_stage2_row
from _tensors import (assert_attention_close, assert_scores_close, dev_bf16, dev_i32, host_bits,
                      score_tolerance)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _index_dev(hi, cfg, M=0, k_mean=None, page=None, sub=None, K=None):
    q, w, k = dev_bf16(hi.q_I), dev_bf16(hi.w_I), dev_bf16(hi.k_I)
    kv, qp = dev_i32(hi.kv_len), dev_i32(hi.q_pos)
    B, T = hi.q_pos.shape
    L_max = hi.k_I.shape[1]
    page = page or cfg.page
    sub = sub or cfg.sub_block
    K = K or cfg.K_sparse
    dbg = torch.full((B, T, L_max), float("nan"), device="cuda")
    pdbg = torch.full((B, T, (L_max + page - 1) // page), float("nan"), device="cuda") if M else None
    ws = torch.empty(lsa.lsa_index_workspace_bytes(B, T, cfg.H_I, cfg.D_I, L_max, K, page, sub, M),
                     dtype=torch.uint8, device="cuda")
    idx = lsa.lsa_index(q, w, k, k_mean, kv, qp, K, cfg.sink, cfg.swa, page, sub, M,
                        scores_dbg=dbg, page_scores_dbg=pdbg, ws=ws)
    err = lsa.lsa_get_error(ws)
    return idx.cpu().numpy(), dbg.cpu().numpy(), (pdbg.cpu().numpy() if M else None), err


def _check_flat_rows(hi, cfg, idx, dbg, K, rows=None, score_sample=None, rng=None):
    B, T = hi.q_pos.shape
    for b in range(B):
        for i in range(T):
            if rows is not None and (b, i) not in rows:
                continue
            t = int(hi.q_pos[b, i])
            (_, _), (_, _), (lo, hi_) = oracle.regions(t, cfg.sink, cfg.swa)
            dom = np.arange(lo, hi_)
            if score_sample and len(dom) > score_sample:
                dom_s = np.sort(rng.choice(dom, score_sample, replace=False))
            else:
                dom_s = dom
            if len(dom_s):
                ref = oracle.scores(hi.q_I[b, i], hi.w_I[b, i], hi.k_I[b], dom_s)
                tol = score_tolerance(hi.q_I[b, i], hi.w_I[b, i], hi.k_I[b][dom_s], ref)
                assert_scores_close(dbg[b, i, dom_s], ref, tol, f"row ({b},{i}) t={t}")
            want, m = oracle.select_query(dbg[b, i], None, t, K, cfg.sink, cfg.swa)
            assert idx[b, i].tolist() == want.tolist(), f"indices row ({b},{i}) t={t}"
            assert m == min(K, max(0, hi_ - lo))


def _attend_and_check(hi, cfg, idx, layer=0, rows=None):
    q, c = dev_bf16(hi.q[layer]), dev_bf16(hi.c_kv[layer])
    kv, qp = dev_i32(hi.kv_len), dev_i32(hi.q_pos)
    idx_d = dev_i32(idx)
    before = idx_d.clone()
    out, lse = lsa.lsa_attend(q, c, idx_d, kv, qp, cfg.sink, cfg.swa, cfg.scale)
    torch.cuda.synchronize()
    assert torch.equal(idx_d, before), "lsa_attend modified its index buffer"
    o = bf16_bits_to_f32(host_bits(out)).reshape(out.shape)
    ls = lse.cpu().numpy()
    if rows is None:
        ro, rl = oracle.attend(hi.q[layer], hi.c_kv[layer], idx, hi.q_pos, cfg.sink, cfg.swa, 512,
                               cfg.scale)
        assert_attention_close(o, ls, ro, rl, "attention")
    else:
        for (b, i) in rows:
            ro, rl = oracle.attend_query(hi.q[layer][b, i], hi.c_kv[layer][b], idx[b, i],
                                         int(hi.q_pos[b, i]), cfg.sink, cfg.swa, 512, cfg.scale)
            assert_attention_close(o[b, i], ls[b, i], ro, rl, f"attention row ({b},{i})")
    return o, ls


def test_tiny_prefill_all_queries():
    """Config: B=1, L=1024, every query 0..1023, H_I=8, d_I=64, K=256=16+128+112, 8 MLA heads."""
    cfg = TINY
    hi = make_host_inputs(cfg)
    idx, dbg, _, err = _index_dev(hi, cfg)
    assert err == 0
    _check_flat_rows(hi, cfg, idx, dbg, cfg.K_sparse)
    # against the oracle's own fp64 selection: same sets up to near-ties
    ref = oracle.index(hi.q_I, hi.w_I, hi.k_I, None, hi.kv_len, hi.q_pos, cfg.K_sparse, cfg.sink,
                       cfg.swa)
    ov = [len(set(a) & set(b) - {-1}) / len(set(b) - {-1})
          for a, b in zip(idx[0].tolist(), ref[0].tolist()) if len(set(b) - {-1})]
    assert np.mean(ov) > 0.99
    _attend_and_check(hi, cfg, idx)


@pytest.fixture(params=["tcgen05", "tcgen05-1q", "legacy"])
def scoring_path(request, monkeypatch):
    """Run a test through the tcgen05 kernels (the multi-query scorer for rows of several
    queries, 128-head attention), through the one-query tcgen05 scorer for every row, and
    through the CUDA-core scorer and mma.sync attention."""
    monkeypatch.delenv("LSA_NO_TCGEN05", raising=False)
    monkeypatch.delenv("LSA_SCORE_ONE_QUERY", raising=False)
    if request.param == "legacy":
        monkeypatch.setenv("LSA_NO_TCGEN05", "1")
    elif request.param == "tcgen05-1q":
        monkeypatch.setenv("LSA_SCORE_ONE_QUERY", "1")
    return request.param


def test_ragged_batch_many_tiles(scoring_path):
    """3 sequences of different lengths in a larger cache, 6 queries each at boundary positions
    (empty dyn, one-token dyn, mid, last), 64 indexer heads of 128 dims, 128 MLA heads."""
    cfg = LsaConfig("ragged", B=3, L=1300, T=6, K=16 + 256 + 100, sink=16, swa=256, n_needles=4,
                    L_max=1400, seed=3)
    kv_len = np.array([1000, 517, 1300], np.int32)
    q_pos = np.array([[0, 10, 271, 272, 600, 999],
                      [516, 300, 15, 16, 290, 500],
                      [1299, 1298, 1000, 273, 700, 1200]], np.int32)
    hi = make_host_inputs(cfg, q_pos=q_pos, kv_len=kv_len)
    idx, dbg, _, err = _index_dev(hi, cfg)
    assert err == 0
    _check_flat_rows(hi, cfg, idx, dbg, cfg.K_sparse)
    assert np.all(idx[0, 0] == -1) and np.all(idx[0, 1] == -1)       # empty dyn
    assert idx[0, 3, 0] == 16 and np.all(idx[0, 3, 1:] == -1)       # dyn = {16}
    _attend_and_check(hi, cfg, idx)


@pytest.mark.parametrize("H_I,T", [(128, 5), (64, 9)])
def test_prefill_rows_share_key_tiles(H_I, T, scoring_path):
    """Several queries of one sequence per call (the multi-query scorer's groups of 256 / H_I
    queries, a short last group) with positions spread over the cache, so the queries of a group
    have dynamic regions of very different lengths; two sequences of different lengths."""
    cfg = LsaConfig("prefill_rows", B=2, L=2500, T=T, H_I=H_I, K=16 + 300 + 200, sink=16,
                    swa=300, n_needles=4, L_max=2600, seed=23, H=16)
    kv_len = np.array([2500, 1777], np.int32)
    rng = np.random.default_rng(23)
    q_pos = np.stack([np.sort(rng.choice(np.arange(int(n)), T, replace=False)) for n in kv_len])
    q_pos[0, -1], q_pos[1, 0] = 2499, 0
    hi = make_host_inputs(cfg, q_pos=q_pos.astype(np.int32), kv_len=kv_len)
    idx, dbg, _, err = _index_dev(hi, cfg)
    assert err == 0
    _check_flat_rows(hi, cfg, idx, dbg, cfg.K_sparse)
    _attend_and_check(hi, cfg, idx)


def test_unaligned_rows_and_odd_sink(scoring_path):
    """Sink 5 and a cache capacity of 1401 tokens: score rows and the start of dyn fall off
    16-byte boundaries differently in every row, so the select pass's scalar head and tail
    run next to its vector body."""
    cfg = LsaConfig("unaligned", B=3, L=1301, T=3, K=5 + 100 + 250, sink=5, swa=100,
                    n_needles=4, L_max=1401, seed=21, H=16)
    kv_len = np.array([1301, 1000, 777], np.int32)
    q_pos = np.array([[1300, 702, 355], [999, 406, 106], [776, 500, 358]], np.int32)
    hi = make_host_inputs(cfg, q_pos=q_pos, kv_len=kv_len)
    idx, dbg, _, err = _index_dev(hi, cfg)
    assert err == 0
    _check_flat_rows(hi, cfg, idx, dbg, cfg.K_sparse)
    _attend_and_check(hi, cfg, idx)


def test_dsa_mode_whole_prefix():
    """sink = swa = 0: plain DSA, K = 2048 over the whole causal prefix (more than some rows)."""
    cfg = LsaConfig("dsa", B=2, L=3000, T=3, K=2048, sink=0, swa=0, n_needles=0, seed=5, H=16)
    q_pos = np.array([[2999, 2047, 100], [2048, 1500, 0]], np.int32)
    hi = make_host_inputs(cfg, q_pos=q_pos)
    idx, dbg, _, err = _index_dev(hi, cfg)
    assert err == 0
    _check_flat_rows(hi, cfg, idx, dbg, 2048)
    assert idx[0, 1].tolist() == list(range(2048))                 # 2048 candidates, K = 2048
    assert idx[1, 2, 0] == 0 and np.all(idx[1, 2, 1:] == -1)
    _attend_and_check(hi, cfg, idx)


def test_ties_go_to_lower_positions():
    """Identical keys give identical scores: the selection is the lowest positions of dyn.
    Keys with every head's dot negative give all-zero scores (ReLU): same rule."""
    cfg = LsaConfig("ties", B=2, L=5000, T=2, K=16 + 64 + 300, sink=16, swa=64, n_needles=0,
                    seed=7, H=8)
    hi = make_host_inputs(cfg, q_pos=np.array([[4999, 3000], [4999, 2000]], np.int32),
                          with_attention=False)
    hi.k_I[0, :] = hi.k_I[0, 123]
    q = bf16_bits_to_f32(hi.q_I[1]).copy()
    q = np.abs(q)
    hi.q_I[1] = to_bf16_bits(q)
    hi.k_I[1] = to_bf16_bits(-np.abs(bf16_bits_to_f32(hi.k_I[1])))
    idx, dbg, _, err = _index_dev(hi, cfg)
    assert err == 0
    for b in range(2):
        for i in range(2):
            t = int(hi.q_pos[b, i])
            assert idx[b, i].tolist() == list(range(16, 16 + 300)), (b, i)
    assert np.all(dbg[1, :, 16:2000 - 63] == 0.0)
    _check_flat_rows(hi, cfg, idx, dbg, cfg.K_sparse)


def _append_all(hi, cfg, chunks):
    """Fill an empty cache through lsa_kv_append in ragged chunks; return device k_I, k_mean."""
    B, L_max, D = hi.k_I.shape
    k = torch.zeros(B, L_max, D, dtype=torch.bfloat16, device="cuda")
    nb = (L_max + cfg.sub_block - 1) // cfg.sub_block
    km = torch.zeros(B, nb, D, dtype=torch.bfloat16, device="cuda")
    src = dev_bf16(hi.k_I)
    errw = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = 0
    for n in chunks:
        old = dev_i32(np.full(B, pos, np.int32))
        lsa.lsa_kv_append(old, k_I_new=src[:, pos:pos + n].contiguous(), k_I=k, k_mean=km,
                          sub_block=cfg.sub_block, device_error=errw)
        pos += n
    torch.cuda.synchronize()
    assert int(errw.item()) == 0
    return k, km


@pytest.mark.parametrize("sub", [8, 128, 1])
def test_append_block_means(sub):
    cfg = LsaConfig("append", B=2, L=1003, T=1, K=100, sink=16, swa=64, n_needles=0, seed=9,
                    sub_block=sub)
    hi = make_host_inputs(cfg, with_attention=False)
    k, km = _append_all(hi, cfg, [1, 7, 500, 3, 492])
    assert np.array_equal(host_bits(k), hi.k_I)
    got = bf16_bits_to_f32(host_bits(km)).astype(np.float64)
    for b in range(2):
        ref = oracle.block_means(hi.k_I[b], 1003, sub)
        g = got[b, :ref.shape[0]]
        # within one bf16 rounding (half an ulp, 2^-8 relative) of the fp64 mean
        step = np.abs(ref) * 2.0 ** -8 + 1e-6
        assert np.all(np.abs(g - ref) <= step), np.abs(g - ref).max()
    # overflow is refused on the device and leaves the cache untouched
    errw = torch.zeros(1, dtype=torch.int32, device="cuda")
    snap = k.clone()
    lsa.lsa_kv_append(dev_i32(np.full(2, 1003, np.int32)), k_I_new=dev_bf16(hi.k_I[:, :5]), k_I=k,
                      k_mean=km, sub_block=sub, device_error=errw)
    torch.cuda.synchronize()
    assert int(errw.item()) == lsa.DEVERR_APPEND and torch.equal(snap, k)


@pytest.mark.parametrize("M,sub", [(6, 8), (3, 128), (64, 8)])
def test_hierarchical_indexing_small(M, sub, scoring_path):
    """HI on a 6000-token cache (ragged last page): page scores within tolerance of Eq. 9 on the
    stored means, the recalled pages and final indices bit-exact when the oracle selects from
    the GPU's page and token scores; with M >= #pages the result equals the flat indexer."""
    cfg = LsaConfig("hi", B=2, L=6000, T=2, K=16 + 512 + 200, sink=16, swa=512, n_needles=8,
                    seed=11, M=M, sub_block=sub, page=128, H=16)
    q_pos = np.array([[5999, 4000], [5999, 700]], np.int32)
    hi = make_host_inputs(cfg, q_pos=q_pos)
    _, km = _append_all(hi, cfg, [6000])
    km_bits = host_bits(km)
    idx, dbg, pdbg, err = _index_dev(hi, cfg, M=M, k_mean=km)
    assert err == 0
    for b in range(2):
        for i in range(2):
            t = int(q_pos[b, i])
            (_, _), (_, _), (lo, hi_) = oracle.regions(t, cfg.sink, cfg.swa)
            pages = np.arange(lo // 128, (hi_ - 1) // 128 + 1)
            ref = np.array([oracle.page_score(hi.q_I[b, i], hi.w_I[b, i], km_bits[b], 6000, 128,
                                              sub, p) for p in pages])
            # tolerance: Eq. 9 sums one Eq. 1 term per sub-block of the page
            per = 128 // sub
            nb = (6000 + sub - 1) // sub
            mags = np.zeros(len(pages))
            for j, p in enumerate(pages):
                ns = np.arange(p * per, min(p * per + per, nb))
                mags[j] = score_tolerance(hi.q_I[b, i], hi.w_I[b, i], km_bits[b][ns],
                                          np.zeros(len(ns))).sum()
            tol = 1e-3 * np.abs(ref) + mags
            assert_scores_close(pdbg[b, i, pages], ref, tol, f"page scores ({b},{i})")
            # stage 2 (Eq. 10): exactly the recalled pages' tokens within dyn are scored, each
            # within tolerance of fp64 Eq. 1
            check_stage2_row(dbg[b, i], pdbg[b, i], hi.q_I[b, i], hi.w_I[b, i], hi.k_I[b], t,
                             cfg.sink, cfg.swa, 128, M, f"row ({b},{i})")
            want, _ = oracle.select_query(dbg[b, i], pdbg[b, i], t, cfg.K_sparse, cfg.sink,
                                          cfg.swa, 128, M)
            assert idx[b, i].tolist() == want.tolist(), (b, i)
    # reported, not gated: overlap with the oracle's own fp64 HI selection
    ref = oracle.index(hi.q_I, hi.w_I, hi.k_I, km_bits, hi.kv_len, hi.q_pos, cfg.K_sparse,
                       cfg.sink, cfg.swa, 128, sub, M)
    ov = [len(set(x) & set(y) - {-1}) / max(1, len(set(y) - {-1}))
          for x, y in zip(idx.reshape(-1, cfg.K_sparse).tolist(),
                          ref.reshape(-1, cfg.K_sparse).tolist())]
    print(f"HI M={M} sub={sub}: overlap with the oracle's fp64 selection {np.mean(ov):.4f}")
    if M >= 6000 // 128 + 1:
        flat, _, _, _ = _index_dev(hi, cfg)
        assert np.array_equal(idx, flat)
    _attend_and_check(hi, cfg, idx)


def test_device_errors_are_flagged_not_trapped():
    cfg = LsaConfig("err", B=1, L=2000, T=2, K=16 + 64 + 50, sink=16, swa=64, n_needles=0,
                    seed=13, H=8)
    hi = make_host_inputs(cfg, q_pos=np.array([[1999, 1500]], np.int32))
    # a query position beyond the sequence: QPOS flag, row returned as -1, others fine
    bad = hi.q_pos.copy()
    bad[0, 1] = 2000
    hi2 = make_host_inputs(cfg, q_pos=bad)
    idx, dbg, _, err = _index_dev(hi2, cfg)
    assert err & lsa.DEVERR_QPOS
    assert np.all(idx[0, 1] == -1)
    # attention with an index inside the window, and one out of order
    idx, _, _, err = _index_dev(hi, cfg)
    assert err == 0
    q, c = dev_bf16(hi.q[0]), dev_bf16(hi.c_kv[0])
    kv, qp = dev_i32(hi.kv_len), dev_i32(hi.q_pos)
    for mutate in ("window", "order"):
        x = idx.copy()
        if mutate == "window":
            x[0, 0, 3] = 1990
        else:
            x[0, 0, 3], x[0, 0, 4] = x[0, 0, 4], x[0, 0, 3]
        ws = torch.empty(lsa.lsa_attend_workspace_bytes(1, 2, 8, 512, 50, 16, 64),
                         dtype=torch.uint8, device="cuda")
        lsa.lsa_attend(q, c, dev_i32(x), kv, qp, cfg.sink, cfg.swa, cfg.scale, ws=ws)
        assert lsa.lsa_get_error(ws) & lsa.DEVERR_INDEX, mutate
    # the context is still usable
    ws = torch.empty(lsa.lsa_attend_workspace_bytes(1, 2, 8, 512, 50, 16, 64), dtype=torch.uint8,
                     device="cuda")
    lsa.lsa_attend(q, c, dev_i32(idx), kv, qp, cfg.sink, cfg.swa, cfg.scale, ws=ws)
    assert lsa.lsa_get_error(ws) == 0


def test_cli_reuse_layer_consumes_owner_indices():
    """Cross-Layer Indexing (N=2): the reuse layer attends with the owner's index buffer, which
    stays byte-identical, over its own queries and latent cache."""
    cfg = LsaConfig("cli", B=2, L=4096, T=1, K=16 + 512 + 300, sink=16, swa=512, n_needles=8,
                    seed=17, layers=2)
    hi = make_host_inputs(cfg)
    idx, _, _, err = _index_dev(hi, cfg)
    assert err == 0
    owner = idx.copy()
    _attend_and_check(hi, cfg, idx, layer=0)
    _attend_and_check(hi, cfg, idx, layer=1)
    assert np.array_equal(idx, owner)


@pytest.mark.parametrize("scale", [1.0 / 24.0, 0.5, 2.0])
def test_attention_wide_logit_range(scale, scoring_path):
    """Large softmax scales make the running max jump by many octaves from tile to tile, which
    exercises the attention kernels' rescaling of the partial output (128 heads)."""
    cfg = LsaConfig("wide", B=2, L=3000, T=3, K=16 + 256 + 300, sink=16, swa=256, n_needles=6,
                    seed=19, scale=scale)
    q_pos = np.array([[2999, 1500, 600], [2999, 2000, 280]], np.int32)
    hi = make_host_inputs(cfg, q_pos=q_pos)
    idx, _, _, err = _index_dev(hi, cfg)
    assert err == 0
    _attend_and_check(hi, cfg, idx)
