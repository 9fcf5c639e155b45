"""Parity at the benchmark's full sizes and launch configuration, on sampled outputs the oracle
can compute one by one: decode 32 x 131072 (CLI pair) and decode 4 x 1048576 (hierarchical and
flat).  Scores are checked on sampled positions; index sets are checked bit-exact by letting the
oracle select from the GPU's full score rows; attention is checked on sampled queries by
gathering their S_t rows (sink, window and selected) into a compact cache."""
import numpy as np
import pytest

import oracle
from lightning_indexer_top_score_b200 import lsa
from lightning_indexer_top_score_b200.workloads import (DECODE_128K, DECODE_1M_HI, DeviceInputs,
                                                        bf16_bits_to_f32)
from _hi_checks import check_stage2_row
from _tensors import assert_attention_close, assert_scores_close, host_bits, score_tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _fill_means(inp, cfg):
    zero = torch.zeros(cfg.B, dtype=torch.int32, device="cuda")
    lsa.lsa_kv_append(zero, k_I_new=inp.k_I[:, :cfg.L].contiguous(), k_I=inp.k_I,
                      k_mean=inp.k_mean, sub_block=cfg.sub_block)


def _key_rows(inp, b):
    """bf16 bits of sequence b's indexer key rows at the given positions (gathered on the
    device, so the full cache is never copied to the host)."""
    return lambda pos: host_bits(inp.k_I[b, torch.from_numpy(np.asarray(pos, np.int64)).cuda()])


def _run_index(inp, cfg, M):
    B, T = cfg.B, cfg.T
    dbg = torch.full((B, T, cfg.cap), float("nan"), device="cuda")
    pdbg = (torch.full((B, T, (cfg.cap + cfg.page - 1) // cfg.page), float("nan"), device="cuda")
            if M else None)
    ws = torch.empty(lsa.lsa_index_workspace_bytes(B, T, cfg.H_I, cfg.D_I, cfg.cap, cfg.K_sparse,
                                                   cfg.page, cfg.sub_block, M),
                     dtype=torch.uint8, device="cuda")
    idx = lsa.lsa_index(inp.q_I, inp.w_I, inp.k_I, inp.k_mean if M else None, inp.kv_len,
                        inp.q_pos, cfg.K_sparse, cfg.sink, cfg.swa, cfg.page, cfg.sub_block, M,
                        scores_dbg=dbg, page_scores_dbg=pdbg, ws=ws)
    assert lsa.lsa_get_error(ws) == 0
    return idx, dbg, pdbg


def _check_row_scores(inp, cfg, b, dbg_row, rng, n=4096):
    t = int(inp.q_pos[b, 0].item())
    (_, _), (_, _), (lo, hi) = oracle.regions(t, cfg.sink, cfg.swa)
    pos = np.sort(rng.choice(np.arange(lo, hi), min(n, hi - lo), replace=False))
    needles = inp.needles[b][inp.needles[b] >= 0] if inp.needles is not None else []
    pos = np.union1d(pos, [p for p in needles if lo <= p < hi]).astype(np.int64)
    kb = host_bits(inp.k_I[b, torch.from_numpy(pos).cuda()])
    q, w = host_bits(inp.q_I[b, 0]), host_bits(inp.w_I[b, 0])
    ref = oracle.scores(q, w, kb, np.arange(len(pos)))
    assert_scores_close(dbg_row[pos], ref, score_tolerance(q, w, kb, ref), f"row {b}")
    return t


def _check_row_attention(inp, cfg, layer, b, idx_row, out, lse):
    t = int(inp.q_pos[b, 0].item())
    (s0, s1), (w0, w1), _ = oracle.regions(t, cfg.sink, cfg.swa)
    rows = np.concatenate([np.arange(s0, s1), np.arange(w0, w1), idx_row[idx_row >= 0]])
    c = host_bits(inp.c_kv[layer][b, torch.from_numpy(rows.astype(np.int64)).cuda()])
    q = host_bits(inp.q[layer][b, 0])
    n = len(rows)
    # a compact cache of the S_t rows, attended as one dynamic set (order does not matter)
    ro, rl = oracle.attend_query(q, c, np.arange(n, dtype=np.int32), n - 1, 0, 0, 512, cfg.scale)
    o = bf16_bits_to_f32(host_bits(out[b, 0])).reshape(cfg.H, 512)
    assert_attention_close(o, lse[b, 0].cpu().numpy(), ro, rl, f"layer {layer} row {b}")


def test_decode_128k_cli_pair_sampled():
    cfg = DECODE_128K
    inp = DeviceInputs(cfg)
    idx, dbg, _ = _run_index(inp, cfg, 0)
    idx_h = idx.cpu().numpy()
    rng = np.random.default_rng(0)
    rows = [0, 17, 31]
    for b in rows:
        row = dbg[b, 0].cpu().numpy()
        t = _check_row_scores(inp, cfg, b, row, rng)
        want, m = oracle.select_query(row, None, t, cfg.K_sparse, cfg.sink, cfg.swa)
        assert idx_h[b, 0].tolist() == want.tolist(), f"indices row {b}"
        assert m == cfg.K_sparse
        # planted needles align with the query: they must be selected
        nd = inp.needles[b][inp.needles[b] >= 0]
        assert np.isin(nd, idx_h[b, 0]).mean() >= 0.95
    ws = torch.empty(lsa.lsa_attend_workspace_bytes(cfg.B, 1, cfg.H, 512, cfg.K_sparse, cfg.sink,
                                                    cfg.swa), dtype=torch.uint8, device="cuda")
    before = idx.clone()
    for layer in range(2):   # owner, then the reuse layer with the owner's indices
        out, lse = lsa.lsa_attend(inp.q[layer], inp.c_kv[layer], idx, inp.kv_len, inp.q_pos,
                                  cfg.sink, cfg.swa, cfg.scale, ws=ws)
        assert lsa.lsa_get_error(ws) == 0
        for b in rows:
            _check_row_attention(inp, cfg, layer, b, idx_h[b, 0], out, lse)
    assert torch.equal(idx, before)


@pytest.mark.parametrize("M", [1024, 0])
def test_decode_1m_sampled(M):
    cfg = DECODE_1M_HI
    inp = DeviceInputs(cfg, with_attention=(M > 0))
    _fill_means(inp, cfg)
    idx, dbg, pdbg = _run_index(inp, cfg, M)
    idx_h = idx.cpu().numpy()
    rng = np.random.default_rng(1)
    for b in (0, 3):
        row = dbg[b, 0].cpu().numpy()
        t = int(inp.q_pos[b, 0].item())
        (_, _), (_, _), (lo, hi) = oracle.regions(t, cfg.sink, cfg.swa)
        if M:
            prow = pdbg[b, 0].cpu().numpy()
            km = host_bits(inp.k_mean[b])
            q, w = host_bits(inp.q_I[b, 0]), host_bits(inp.w_I[b, 0])
            pages = np.arange(lo // cfg.page, (hi - 1) // cfg.page + 1)
            for p in rng.choice(pages, 64, replace=False):
                ref = oracle.page_score(q, w, km, cfg.L, cfg.page, cfg.sub_block, int(p))
                per = cfg.page // cfg.sub_block
                mag = score_tolerance(q, w, km[p * per:(p + 1) * per], np.zeros(per)).sum()
                assert abs(prow[p] - ref) <= 1e-3 * abs(ref) + mag, (b, p)
            want, _ = oracle.select_query(row, prow, t, cfg.K_sparse, cfg.sink, cfg.swa,
                                          cfg.page, M)
            # stage 2 (Eq. 10): scored tokens are exactly the recalled pages' tokens within dyn;
            # sampled ones against fp64 Eq. 1
            check_stage2_row(row, prow, q, w, _key_rows(inp, b), t, cfg.sink, cfg.swa, cfg.page,
                             M, f"row {b}", sample=4096, rng=rng)
        else:
            _check_row_scores(inp, cfg, b, row, rng)
            want, _ = oracle.select_query(row, None, t, cfg.K_sparse, cfg.sink, cfg.swa)
        assert idx_h[b, 0].tolist() == want.tolist(), f"indices row {b} M={M}"
    if M:
        ws = torch.empty(lsa.lsa_attend_workspace_bytes(cfg.B, 1, cfg.H, 512, cfg.K_sparse,
                                                        cfg.sink, cfg.swa),
                         dtype=torch.uint8, device="cuda")
        out, lse = lsa.lsa_attend(inp.q[0], inp.c_kv[0], idx, inp.kv_len, inp.q_pos, cfg.sink,
                                  cfg.swa, cfg.scale, ws=ws)
        assert lsa.lsa_get_error(ws) == 0
        for b in (0, 3):
            _check_row_attention(inp, cfg, 0, b, idx_h[b, 0], out, lse)


@pytest.mark.parametrize("L,variant", [(1048576, "dsa"), (262144, "lsa"), (524288, "lsa")])
def test_sweep_point_sampled(L, variant):
    """Points of the paper's length table (Table 1 shape, batch 8, decode) that no other test
    covers: the DSA-style flat top-2048 over a whole 1M-token prefix (no sink or window), and
    LSA with hierarchical indexing at 256K and 512K (P = 128, 8-token sub-blocks, M = 1024)
    followed by both layers of the CLI pair.  Sampled scores (stage-2 scores and the exact
    scored set for HI, sampled page scores against Eq. 9), selection bit-exact by the oracle from
    the GPU's score rows, and attention of two rows per layer."""
    from lightning_indexer_top_score_b200.workloads import sweep_config
    cfg = sweep_config(L, variant)
    inp = DeviceInputs(cfg)
    M = cfg.M
    if M:
        _fill_means(inp, cfg)
    idx, dbg, pdbg = _run_index(inp, cfg, M)
    idx_h = idx.cpu().numpy()
    rng = np.random.default_rng(9)
    rows = (0, cfg.B - 1)
    per = cfg.page // cfg.sub_block
    for b in rows:
        row = dbg[b, 0].cpu().numpy()
        t = int(inp.q_pos[b, 0].item())
        if M:
            prow = pdbg[b, 0].cpu().numpy()
            km = host_bits(inp.k_mean[b])
            q, w = host_bits(inp.q_I[b, 0]), host_bits(inp.w_I[b, 0])
            (_, _), (_, _), (lo, hi) = oracle.regions(t, cfg.sink, cfg.swa)
            pages = np.arange(lo // cfg.page, (hi - 1) // cfg.page + 1)
            for p in rng.choice(pages, 32, replace=False):
                ref = oracle.page_score(q, w, km, cfg.L, cfg.page, cfg.sub_block, int(p))
                mag = score_tolerance(q, w, km[p * per:(p + 1) * per], np.zeros(per)).sum()
                assert abs(prow[p] - ref) <= 1e-3 * abs(ref) + mag, (b, p)
            check_stage2_row(row, prow, q, w, _key_rows(inp, b), t, cfg.sink, cfg.swa, cfg.page,
                             M, f"row {b}", sample=4096, rng=rng)
            want, m = oracle.select_query(row, prow, t, cfg.K_sparse, cfg.sink, cfg.swa,
                                          cfg.page, M)
        else:
            _check_row_scores(inp, cfg, b, row, rng)
            want, m = oracle.select_query(row, None, t, cfg.K_sparse, cfg.sink, cfg.swa)
        assert m == cfg.K_sparse
        assert idx_h[b, 0].tolist() == want.tolist(), f"indices row {b}"
    ws = torch.empty(lsa.lsa_attend_workspace_bytes(cfg.B, 1, cfg.H, 512, cfg.K_sparse, cfg.sink,
                                                    cfg.swa), dtype=torch.uint8, device="cuda")
    for layer in range(cfg.layers):
        out, lse = lsa.lsa_attend(inp.q[layer], inp.c_kv[layer], idx, inp.kv_len, inp.q_pos,
                                  cfg.sink, cfg.swa, cfg.scale, ws=ws)
        assert lsa.lsa_get_error(ws) == 0
        for b in rows:
            _check_row_attention(inp, cfg, layer, b, idx_h[b, 0], out, lse)


def test_prefill_32k_chunk_sampled():
    """Chunked causal prefill, L = 32768 with clustered topics: the last 4096-query chunk (the
    bench's launch configuration) -- sampled scores, exact selection from the GPU's score rows,
    and attention of sampled queries."""
    from dataclasses import replace
    from lightning_indexer_top_score_b200.workloads import PREFILL_32K
    cfg = PREFILL_32K
    inp = DeviceInputs(cfg)
    C = cfg.chunk
    a, b = cfg.L - C, cfg.L
    q_I = inp.q_I[:, a:b].contiguous()
    w_I = inp.w_I[:, a:b].contiguous()
    q = inp.q[0][:, a:b].contiguous()
    qp = torch.arange(a, b, dtype=torch.int32, device="cuda").view(1, -1).contiguous()
    dbg = torch.full((1, C, cfg.cap), float("nan"), device="cuda")
    ws = torch.empty(lsa.lsa_index_workspace_bytes(1, C, cfg.H_I, cfg.D_I, cfg.cap, cfg.K_sparse),
                     dtype=torch.uint8, device="cuda")
    idx = lsa.lsa_index(q_I, w_I, inp.k_I, None, inp.kv_len, qp, cfg.K_sparse, cfg.sink, cfg.swa,
                        scores_dbg=dbg, ws=ws)
    assert lsa.lsa_get_error(ws) == 0
    out, lse = lsa.lsa_attend(q, inp.c_kv[0], idx, inp.kv_len, qp, cfg.sink, cfg.swa, cfg.scale)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    rows = [0, 1, C // 2, C - 1] + list(rng.choice(C, 4, replace=False))
    idx_h = idx[0].cpu().numpy()
    for i in rows:
        t = a + int(i)
        row = dbg[0, i].cpu().numpy()
        (_, _), (_, _), (lo, hi) = oracle.regions(t, cfg.sink, cfg.swa)
        pos = np.sort(rng.choice(np.arange(lo, hi), 2048, replace=False)).astype(np.int64)
        kb = host_bits(inp.k_I[0, torch.from_numpy(pos).cuda()])
        qh, wh = host_bits(q_I[0, i]), host_bits(w_I[0, i])
        ref = oracle.scores(qh, wh, kb, np.arange(len(pos)))
        assert_scores_close(row[pos], ref, score_tolerance(qh, wh, kb, ref), f"query {t}")
        want, _ = oracle.select_query(row, None, t, cfg.K_sparse, cfg.sink, cfg.swa)
        assert idx_h[i].tolist() == want.tolist(), f"indices query {t}"
        (s0, s1), (w0, w1), _ = oracle.regions(t, cfg.sink, cfg.swa)
        sel = idx_h[i]
        keys = np.concatenate([np.arange(s0, s1), np.arange(w0, w1), sel[sel >= 0]])
        c = host_bits(inp.c_kv[0][0, torch.from_numpy(keys.astype(np.int64)).cuda()])
        ro, rl = oracle.attend_query(host_bits(q[0, i]), c, np.arange(len(keys), dtype=np.int32),
                                     len(keys) - 1, 0, 0, 512, cfg.scale)
        o = bf16_bits_to_f32(host_bits(out[0, i])).reshape(cfg.H, 512)
        assert_attention_close(o, lse[0, i].cpu().numpy(), ro, rl, f"attention query {t}")


def test_index_chunk_hi_256k_sampled():
    """Hierarchical indexer on one prefill chunk, the paper's Table 4 setting at the 256K gate:
    the last 2048 queries of a 262144-token sequence, P = 128, 8-token sub-blocks, M = 1024.
    Sampled page scores against Eq. 9 on the stored means; exact selection of sampled queries
    by the oracle from the GPU's page and token score rows; scored tokens stay within the
    recalled pages and dyn."""
    from lightning_indexer_top_score_b200.workloads import index_chunk_config
    cfg = index_chunk_config(262144, "hi")
    inp = DeviceInputs(cfg, with_attention=False)
    _fill_means(inp, cfg)
    M = cfg.M
    idx, dbg, pdbg = _run_index(inp, cfg, M)
    idx_h = idx[0].cpu().numpy()
    km = host_bits(inp.k_mean[0])
    rng = np.random.default_rng(5)
    per = cfg.page // cfg.sub_block
    for i in [0, 1, cfg.T // 2, cfg.T - 1] + list(rng.choice(cfg.T, 2, replace=False)):
        i = int(i)
        t = int(inp.q_pos[0, i].item())
        row = dbg[0, i].cpu().numpy()
        prow = pdbg[0, i].cpu().numpy()
        (_, _), (_, _), (lo, hi) = oracle.regions(t, cfg.sink, cfg.swa)
        q, w = host_bits(inp.q_I[0, i]), host_bits(inp.w_I[0, i])
        pages = np.arange(lo // cfg.page, (hi - 1) // cfg.page + 1)
        for pg in rng.choice(pages, 16, replace=False):
            ref = oracle.page_score(q, w, km, cfg.L, cfg.page, cfg.sub_block, int(pg))
            mag = score_tolerance(q, w, km[pg * per:(pg + 1) * per], np.zeros(per)).sum()
            assert abs(prow[pg] - ref) <= 1e-3 * abs(ref) + mag, (i, pg)
        check_stage2_row(row, prow, q, w, _key_rows(inp, 0), t, cfg.sink, cfg.swa, cfg.page, M,
                         f"query {t}", sample=2048, rng=rng)
        want, _ = oracle.select_query(row, prow, t, cfg.K_sparse, cfg.sink, cfg.swa, cfg.page, M)
        assert idx_h[i].tolist() == want.tolist(), f"indices query {t}"


def test_train_8k_backward_sampled():
    """The training workload at its full size (the paper's Table 2 setting: 8192 queries over an
    8192-token sequence, 128 heads, K = 2048), forward then backward from the forward's out / lse
    as the bench runs them.  Checked against the oracle: dq of sampled queries (a query's dq
    depends on its own row only), and the gradient rows of the last four positions.  Those rows
    lie in no dynamic region (it ends at t - 1024), so only the windows of the queries at or
    after them reach them, and the oracle sums those few queries exactly."""
    import torch
    from _bwd_bounds import assert_grad_close, keys_of, row_bounds
    from lightning_indexer_top_score_b200.workloads import bf16_bits_to_f32, train_config
    cfg = train_config(8192)
    inp = DeviceInputs(cfg)
    T = cfg.T
    idx = torch.empty(1, T, cfg.K_sparse, dtype=torch.int32, device="cuda")
    ws_i = torch.empty(lsa.lsa_index_workspace_bytes(1, 512, cfg.H_I, cfg.D_I, cfg.cap,
                                                     cfg.K_sparse, cfg.page, cfg.sub_block, 0),
                       dtype=torch.uint8, device="cuda")
    for a in range(0, T, 512):
        lsa.lsa_index(inp.q_I[:, a:a + 512], inp.w_I[:, a:a + 512], inp.k_I, None, inp.kv_len,
                      inp.q_pos[:, a:a + 512], cfg.K_sparse, cfg.sink, cfg.swa,
                      indices=idx[:, a:a + 512], ws=ws_i)
    assert lsa.lsa_get_error(ws_i) == 0
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    dout = torch.randn(1, T, cfg.H, 512, generator=g, device="cuda").to(torch.bfloat16)
    out, lse = lsa.lsa_attend(inp.q[0], inp.c_kv[0], idx, inp.kv_len, inp.q_pos, cfg.sink,
                              cfg.swa, cfg.scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dc = lsa.lsa_attend_bwd(inp.q[0], inp.c_kv[0], idx, inp.kv_len, inp.q_pos, cfg.sink,
                                cfg.swa, cfg.scale, dout, out=out, lse=lse, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    c_bits = host_bits(inp.c_kv[0][0])
    c = bf16_bits_to_f32(c_bits).astype(np.float64)
    idx_h = idx.cpu().numpy()[0]
    dq_h = dq[0].cpu().numpy()
    last = range(T - 4, T)
    dc_ref = np.zeros((4, 576))
    dc_bound = np.zeros((4, 576))
    for t in [0, 1, 2047, 4096] + list(last):
        q_bits = host_bits(inp.q[0][0, t])
        dout_f = bf16_bits_to_f32(host_bits(dout[0, t])).astype(np.float64)
        dq_ref, dc_seq = oracle.attend_bwd_query(q_bits, c_bits, idx_h[t], t, cfg.sink, cfg.swa,
                                                 512, cfg.scale, dout_f)
        keys = keys_of(t, idx_h[t], cfg.sink, cfg.swa)
        b_dq, b_rows = row_bounds(bf16_bits_to_f32(q_bits).astype(np.float64), c, keys, dout_f,
                                  cfg.scale, True)
        assert_grad_close(dq_h[t], dq_ref, b_dq, f"dq of query {t}")
        if t in last:
            dc_ref += dc_seq[T - 4:]
            for j, s in enumerate(keys):
                if s >= T - 4:
                    dc_bound[s - (T - 4)] += b_rows[j]
    assert_grad_close(dc[0, T - 4:].cpu().numpy(), dc_ref, dc_bound, "dc of the last 4 rows")
