"""MinMax pooling of Hierarchical Indexing stage 1 (LongCat Sparse Attention, Sec. 5.3.5 pooling
ablation, Table 11) through the C-ABI: the MinMax rows kept by lsa_kv_minmax equal the oracle's
element-wise extremes bit for bit; lsa_index_minmax's page scores are within tolerance of the
oracle's MinMax page score on the stored rows; its stage-2 scores cover exactly the recalled
pages within dyn, each within tolerance of fp64 Eq. 1; its indices are bit-exact when the oracle
selects from the GPU's own page and token scores; with every page recalled it equals the flat
indexer."""
import numpy as np
import pytest

import oracle
from lightning_indexer_top_score_b200 import lsa
from lightning_indexer_top_score_b200.workloads import (DeviceInputs, LsaConfig, bf16_bits_to_f32,
                                                        make_host_inputs)
from _hi_checks import check_stage2_row
from _tensors import dev_bf16, dev_i32, host_bits, score_tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _fill(k_src, B, L, D, sub, chunks, L_max=None):
    """Append the keys in ragged chunks through lsa_kv_append, refreshing the MinMax rows after
    each chunk; returns (k_I, k_minmax) on the device."""
    L_max = L_max or L
    k = torch.zeros(B, L_max, D, dtype=torch.bfloat16, device="cuda")
    nb = (L_max + sub - 1) // sub
    kmm = torch.zeros(B, nb, 2 * D, dtype=torch.bfloat16, device="cuda")
    errw = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = 0
    for n in chunks:
        old = dev_i32(np.full(B, pos, np.int32))
        lsa.lsa_kv_append(old, k_I_new=k_src[:, pos:pos + n].contiguous(), k_I=k,
                          device_error=errw)
        lsa.lsa_kv_minmax(old, n, k, kmm, sub_block=sub, device_error=errw)
        pos += n
    torch.cuda.synchronize()
    assert int(errw.item()) == 0
    return k, kmm


def _minmax_tolerance(q, w, rows, D):
    """Per sub-block: 1e-5 * sum_j |w_j| sum_d |q_jd| max(|k_max_d|, |k_min_d|), the size of the
    products the contraction sums (the score rule applied to the larger extreme)."""
    r = bf16_bits_to_f32(rows).astype(np.float64)
    big = np.maximum(np.abs(r[:, :D]), np.abs(r[:, D:]))
    qa = np.abs(bf16_bits_to_f32(q).astype(np.float64))
    wa = np.abs(bf16_bits_to_f32(w).astype(np.float64))
    return 1e-5 * (big @ (wa @ qa))


@pytest.mark.parametrize("sub", [1, 8, 128])
def test_kv_minmax_rows_bit_exact(sub):
    cfg = LsaConfig("mm_rows", B=2, L=1003, T=1, K=100, sink=16, swa=64, n_needles=0, seed=31,
                    sub_block=sub)
    hi = make_host_inputs(cfg, with_attention=False)
    _, kmm = _fill(dev_bf16(hi.k_I), 2, 1003, 128, sub, [1, 7, 500, 3, 492])
    got = host_bits(kmm)
    for b in range(2):
        ref = oracle.block_minmax(hi.k_I[b], 1003, sub)
        assert np.array_equal(bf16_bits_to_f32(got[b, :ref.shape[0]]).astype(np.float64), ref)
    # overflow is refused on the device and leaves the rows untouched
    errw = torch.zeros(1, dtype=torch.int32, device="cuda")
    snap = kmm.clone()
    k = torch.zeros(2, 1003, 128, dtype=torch.bfloat16, device="cuda")
    lsa.lsa_kv_minmax(dev_i32(np.full(2, 1000, np.int32)), 5, k, kmm, sub_block=sub,
                      device_error=errw)
    torch.cuda.synchronize()
    assert int(errw.item()) == lsa.DEVERR_APPEND and torch.equal(snap, kmm)


def _index_minmax(hi, cfg, k, kmm, M, sub):
    B, T = hi.q_pos.shape
    L_max = k.shape[1]
    dbg = torch.full((B, T, L_max), float("nan"), device="cuda")
    pdbg = torch.full((B, T, (L_max + cfg.page - 1) // cfg.page), float("nan"), device="cuda")
    ws = torch.empty(lsa.lsa_index_workspace_bytes(B, T, cfg.H_I, cfg.D_I, L_max, cfg.K_sparse,
                                                   cfg.page, sub, M),
                     dtype=torch.uint8, device="cuda")
    idx = lsa.lsa_index_minmax(dev_bf16(hi.q_I), dev_bf16(hi.w_I), k, kmm, dev_i32(hi.kv_len),
                               dev_i32(hi.q_pos), cfg.K_sparse, cfg.sink, cfg.swa, cfg.page, sub,
                               M, scores_dbg=dbg, page_scores_dbg=pdbg, ws=ws)
    err = lsa.lsa_get_error(ws)
    return idx.cpu().numpy(), dbg.cpu().numpy(), pdbg.cpu().numpy(), err


@pytest.mark.parametrize("M,sub,H_I,D_I", [(6, 8, 64, 128), (3, 32, 128, 128), (5, 4, 64, 64),
                                           (64, 8, 64, 128)])
def test_minmax_hierarchical_indexing_small(M, sub, H_I, D_I):
    cfg = LsaConfig("mm_hi", B=2, L=6000, T=2, K=16 + 512 + 200, sink=16, swa=512, n_needles=8,
                    seed=33, M=M, sub_block=sub, page=128, H_I=H_I, D_I=D_I, H=16)
    q_pos = np.array([[5999, 4000], [5999, 700]], np.int32)
    hi = make_host_inputs(cfg, q_pos=q_pos, with_attention=False)
    k, kmm = _fill(dev_bf16(hi.k_I), 2, 6000, D_I, sub, [6000])
    rows = host_bits(kmm)
    idx, dbg, pdbg, err = _index_minmax(hi, cfg, k, kmm, M, sub)
    assert err == 0
    per = 128 // sub
    nb = (6000 + sub - 1) // sub
    for b in range(2):
        for i in range(2):
            t = int(q_pos[b, i])
            (_, _), (_, _), (lo, hi_) = oracle.regions(t, cfg.sink, cfg.swa)
            pages = np.arange(lo // 128, (hi_ - 1) // 128 + 1)
            q, w = hi.q_I[b, i], hi.w_I[b, i]
            ref = np.array([oracle.page_score_minmax(q, w, rows[b], 6000, 128, sub, int(p))
                            for p in pages])
            mag = _minmax_tolerance(q, w, rows[b][:nb], D_I)
            tol = 1e-3 * np.abs(ref) + np.array(
                [mag[p * per:min(nb, p * per + per)].sum() for p in pages])
            err_p = np.abs(pdbg[b, i, pages].astype(np.float64) - ref)
            assert np.all(err_p <= tol), f"page scores ({b},{i}): worst {err_p.max():.3e}"
            check_stage2_row(dbg[b, i], pdbg[b, i], q, w, hi.k_I[b], t, cfg.sink, cfg.swa, 128, M,
                             f"row ({b},{i})")
            want, _ = oracle.select_query(dbg[b, i], pdbg[b, i], t, cfg.K_sparse, cfg.sink,
                                          cfg.swa, 128, M)
            assert idx[b, i].tolist() == want.tolist(), (b, i)
    if M >= 6000 // 128 + 1:
        flat = lsa.lsa_index(dev_bf16(hi.q_I), dev_bf16(hi.w_I), k, None, dev_i32(hi.kv_len),
                             dev_i32(hi.q_pos), cfg.K_sparse, cfg.sink, cfg.swa).cpu().numpy()
        assert np.array_equal(idx, flat)
    # reported, not gated: overlap with the oracle's own fp64 MinMax selection
    ref = oracle.index(hi.q_I, hi.w_I, hi.k_I, rows, hi.kv_len, hi.q_pos, cfg.K_sparse, cfg.sink,
                       cfg.swa, 128, sub, M, pooling="minmax")
    ov = [len(set(x) & set(y) - {-1}) / max(1, len(set(y) - {-1}))
          for x, y in zip(idx.reshape(-1, cfg.K_sparse).tolist(),
                          ref.reshape(-1, cfg.K_sparse).tolist())]
    print(f"MinMax HI M={M} sub={sub}: overlap with the oracle's fp64 selection {np.mean(ov):.4f}")


def test_minmax_refuses_what_it_does_not_run():
    cfg = LsaConfig("mm_refuse", B=1, L=2048, T=1, K=16 + 64 + 100, sink=16, swa=64,
                    n_needles=0, seed=35, H_I=16, D_I=64, H=8)
    hi = make_host_inputs(cfg, with_attention=False)
    k, kmm = _fill(dev_bf16(hi.k_I), 1, 2048, 64, 8, [2048])
    with pytest.raises(lsa.LsaError) as e:   # 16 indexer heads: no tensor-core scorer
        lsa.lsa_index_minmax(dev_bf16(hi.q_I), dev_bf16(hi.w_I), k, kmm, dev_i32(hi.kv_len),
                             dev_i32(hi.q_pos), cfg.K_sparse, 16, 64, 128, 8, 4)
    assert e.value.status == 2
    with pytest.raises(lsa.LsaError) as e:   # MinMax is a stage-1 pooling: M must be >= 1
        lsa.lsa_index_minmax(dev_bf16(hi.q_I), dev_bf16(hi.w_I), k, kmm, dev_i32(hi.kv_len),
                             dev_i32(hi.q_pos), cfg.K_sparse, 16, 64, 128, 8, 0)
    assert e.value.status == 1


def test_minmax_table11_setting_sampled():
    """The pooling ablation's setting (Table 11): 128K-token decode, M = 128 recalled pages of
    128 tokens, sub-blocks of 8, here over 8 sequences of the decode workload's recipe.  Sampled
    page scores, the exact stage-2 scored set with sampled scores, and the selection bit-exact
    from the GPU's score rows."""
    from dataclasses import replace
    from lightning_indexer_top_score_b200.workloads import DECODE_128K
    cfg = replace(DECODE_128K, B=8, M=128, name="mm_table11")
    inp = DeviceInputs(cfg, with_attention=False)
    nb = (cfg.cap + cfg.sub_block - 1) // cfg.sub_block
    kmm = torch.zeros(cfg.B, nb, 2 * cfg.D_I, dtype=torch.bfloat16, device="cuda")
    lsa.lsa_kv_minmax(torch.zeros(cfg.B, dtype=torch.int32, device="cuda"), cfg.L, inp.k_I, kmm,
                      sub_block=cfg.sub_block)
    B = cfg.B
    dbg = torch.full((B, 1, cfg.cap), float("nan"), device="cuda")
    pdbg = torch.full((B, 1, (cfg.cap + 127) // 128), float("nan"), device="cuda")
    ws = torch.empty(lsa.lsa_index_workspace_bytes(B, 1, cfg.H_I, cfg.D_I, cfg.cap, cfg.K_sparse,
                                                   128, cfg.sub_block, cfg.M),
                     dtype=torch.uint8, device="cuda")
    idx = lsa.lsa_index_minmax(inp.q_I, inp.w_I, inp.k_I, kmm, inp.kv_len, inp.q_pos,
                               cfg.K_sparse, cfg.sink, cfg.swa, 128, cfg.sub_block, cfg.M,
                               scores_dbg=dbg, page_scores_dbg=pdbg, ws=ws)
    assert lsa.lsa_get_error(ws) == 0
    idx_h = idx.cpu().numpy()
    rng = np.random.default_rng(37)
    per = 128 // cfg.sub_block
    for b in (0, B - 1):
        t = int(inp.q_pos[b, 0].item())
        row, prow = dbg[b, 0].cpu().numpy(), pdbg[b, 0].cpu().numpy()
        q, w = host_bits(inp.q_I[b, 0]), host_bits(inp.w_I[b, 0])
        rows = host_bits(kmm[b])
        (_, _), (_, _), (lo, hi) = oracle.regions(t, cfg.sink, cfg.swa)
        pages = np.arange(lo // 128, (hi - 1) // 128 + 1)
        mag = _minmax_tolerance(q, w, rows, cfg.D_I)
        for p in rng.choice(pages, 64, replace=False):
            ref = oracle.page_score_minmax(q, w, rows, cfg.L, 128, cfg.sub_block, int(p))
            assert abs(prow[p] - ref) <= 1e-3 * abs(ref) + mag[p * per:(p + 1) * per].sum(), (b, p)
        check_stage2_row(row, prow, q, w,
                         lambda pos: host_bits(inp.k_I[b, torch.from_numpy(
                             np.asarray(pos, np.int64)).cuda()]),
                         t, cfg.sink, cfg.swa, 128, cfg.M, f"row {b}", sample=4096, rng=rng)
        want, _ = oracle.select_query(row, prow, t, cfg.K_sparse, cfg.sink, cfg.swa, 128, cfg.M)
        assert idx_h[b, 0].tolist() == want.tolist(), f"indices row {b}"
