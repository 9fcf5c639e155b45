"""HFA backward (lsa_attend_bwd) through the C-ABI against the fp64 oracle.

The index sets come from the oracle's own indexer on the same host inputs.  The tolerance is
derived from the kernel's arithmetic in _bwd_bounds: bf16 rounding of p and scale dz before the
gradient products, fp32 sums, and the cancellation in dp_s - D where attention is flat over
identical rows (the planted needles repeat one row), bounded relative to the size of the terms
rather than the result.  test_bwd_bound checks that this bound admits the rounding and rejects a
dropped D, a flipped term and rows one off.
"""
import numpy as np
import pytest

import oracle
from lightning_indexer_top_score_b200 import lsa
from lightning_indexer_top_score_b200.workloads import (LsaConfig, bf16_bits_to_f32,
                                                        make_host_inputs, to_bf16_bits)
from _bwd_bounds import assert_grad_close as _assert_grad_close, keys_of as _keys_of, \
    row_bounds as _row_bounds
from _tensors import dev_bf16, dev_i32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _run(hi, cfg, idx, dout_bits, fwd_outputs):
    """lsa_attend_bwd on device copies; with fwd_outputs, lsa_attend runs first and the backward
    takes its out / lse (the training path)."""
    q, c = dev_bf16(hi.q[0]), dev_bf16(hi.c_kv[0])
    idx_d, kv, qp = dev_i32(idx), dev_i32(hi.kv_len), dev_i32(hi.q_pos)
    out = lse = None
    if fwd_outputs:
        out, lse = lsa.lsa_attend(q, c, idx_d, kv, qp, cfg.sink, cfg.swa, cfg.scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dc = lsa.lsa_attend_bwd(q, c, idx_d, kv, qp, cfg.sink, cfg.swa, cfg.scale,
                                dev_bf16(dout_bits), out=out, lse=lse, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return dq.cpu().numpy(), dc.cpu().numpy()


def _path(monkeypatch, mma_sync):
    """LSA_NO_TCGEN05=1 selects the mma.sync kernels, else the tcgen05 backward runs wherever it
    applies (64-head groups with the forward's out and lse)."""
    monkeypatch.delenv("LSA_NO_TCGEN05", raising=False)
    if mma_sync:
        monkeypatch.setenv("LSA_NO_TCGEN05", "1")


@pytest.mark.parametrize("fwd_outputs,H,mma_sync", [(False, 32, False), (True, 32, False),
                                                    (True, 64, False), (True, 64, True)])
def test_attend_bwd_ragged_shared_rows(fwd_outputs, H, mma_sync, monkeypatch):
    """Three sequences in a larger cache, six queries each (window rows shared between queries,
    so their gradients accumulate; t = 0 has one key), 32 heads (the mma.sync kernel) or 64
    heads (the tcgen05 kernel given the forward's outputs: 128-key tiles with ragged tails)."""
    _path(monkeypatch, mma_sync)
    cfg = LsaConfig("bwd", B=3, L=1300, T=6, K=16 + 256 + 100, sink=16, swa=256, n_needles=4,
                    L_max=1400, seed=41, H=H)
    kv_len = np.array([1000, 517, 1300], np.int32)
    q_pos = np.array([[0, 10, 271, 272, 600, 999],
                      [516, 300, 15, 16, 290, 500],
                      [1299, 1298, 1000, 273, 700, 1200]], np.int32)
    hi = make_host_inputs(cfg, q_pos=q_pos, kv_len=kv_len)
    idx = oracle.index(hi.q_I, hi.w_I, hi.k_I, None, hi.kv_len, hi.q_pos, cfg.K_sparse, cfg.sink,
                       cfg.swa)
    rng = np.random.default_rng(5)
    dout = to_bf16_bits(rng.standard_normal((3, 6, cfg.H, 512)).astype(np.float32))
    dout_f = bf16_bits_to_f32(dout).astype(np.float64)
    dq, dc = _run(hi, cfg, idx, dout, fwd_outputs)
    dq_ref, dc_ref = oracle.attend_bwd(hi.q[0], hi.c_kv[0], idx, hi.q_pos, cfg.sink, cfg.swa, 512,
                                       cfg.scale, dout_f)
    q = bf16_bits_to_f32(hi.q[0]).astype(np.float64)
    c = bf16_bits_to_f32(hi.c_kv[0]).astype(np.float64)
    m_dq = np.zeros_like(dq_ref)
    m_dc = np.zeros_like(dc_ref)
    for b in range(3):
        for i in range(6):
            keys = _keys_of(int(q_pos[b, i]), idx[b, i], cfg.sink, cfg.swa)
            m_dq[b, i], rows = _row_bounds(q[b, i], c[b], keys, dout_f[b, i], cfg.scale,
                                            fwd_outputs)
            np.add.at(m_dc[b], keys, rows)
    assert not dq_ref[0, 0].any()
    if not fwd_outputs:
        assert not dq[0, 0].any()  # one key: p = 1 and D = dp exactly, so dz = 0
    _assert_grad_close(dq, dq_ref, m_dq, "dq")
    touched = m_dc.sum(axis=-1) > 0
    _assert_grad_close(dc[touched], dc_ref[touched], m_dc[touched], "dc (rows of some S_t)")
    assert not dc[~touched].any(), "gradient written to a row outside every S_t"


@pytest.mark.parametrize("fwd_outputs,mma_sync", [(False, False), (True, False), (True, True)])
def test_attend_bwd_decode_128_heads_sampled(fwd_outputs, mma_sync, monkeypatch):
    """128 heads (two tcgen05 head groups or four mma.sync ones per query), 4 sequences of 16384
    tokens, one query each, K = 2048 (16 + 1024 + 1008); two sequences checked in full (dq and
    every row gradient)."""
    _path(monkeypatch, mma_sync)
    cfg = LsaConfig("bwd_decode", B=4, L=16384, T=1, n_needles=8, seed=43)
    hi = make_host_inputs(cfg)
    idx = oracle.index(hi.q_I, hi.w_I, hi.k_I, None, hi.kv_len, hi.q_pos, cfg.K_sparse, cfg.sink,
                       cfg.swa)
    rng = np.random.default_rng(6)
    dout = to_bf16_bits(rng.standard_normal((4, 1, cfg.H, 512)).astype(np.float32))
    dq, dc = _run(hi, cfg, idx, dout, fwd_outputs)
    for b in (0, 3):
        t = int(hi.q_pos[b, 0])
        dout_f = bf16_bits_to_f32(dout[b, 0]).astype(np.float64)
        dq_ref, dc_ref = oracle.attend_bwd_query(hi.q[0][b, 0], hi.c_kv[0][b], idx[b, 0], t,
                                                 cfg.sink, cfg.swa, 512, cfg.scale, dout_f)
        keys = _keys_of(t, idx[b, 0], cfg.sink, cfg.swa)
        assert len(keys) == 2048
        m_dq, rows = _row_bounds(bf16_bits_to_f32(hi.q[0][b, 0]).astype(np.float64),
                                 bf16_bits_to_f32(hi.c_kv[0][b]).astype(np.float64), keys, dout_f,
                                 cfg.scale, fwd_outputs)
        _assert_grad_close(dq[b, 0], dq_ref, m_dq, f"dq sequence {b}")
        _assert_grad_close(dc[b][keys], dc_ref[keys], rows, f"dc sequence {b}")
        others = np.ones(dc.shape[1], bool)
        others[keys] = False
        assert not dc[b][others].any()


@pytest.mark.parametrize("mma_sync", [False, True])
def test_attend_bwd_dsa_mode_64_heads(mma_sync, monkeypatch):
    """DSA mode (no sink, no window: every key is a gathered pick), 64 heads (one tcgen05 head
    group or two mma.sync ones), ragged lengths, K = 2100 (for the mma.sync kernel an index row
    longer than its shared-memory copy, so the positions are read from the caller's buffer)."""
    _path(monkeypatch, mma_sync)
    cfg = LsaConfig("bwd_dsa", B=2, L=3000, T=3, K=2100, sink=0, swa=0, n_needles=4, seed=47,
                    H=64)
    kv_len = np.array([3000, 1600], np.int32)
    q_pos = np.array([[100, 2000, 2999], [50, 199, 1599]], np.int32)
    hi = make_host_inputs(cfg, q_pos=q_pos, kv_len=kv_len)
    idx = oracle.index(hi.q_I, hi.w_I, hi.k_I, None, hi.kv_len, hi.q_pos, cfg.K_sparse, 0, 0)
    rng = np.random.default_rng(8)
    dout = to_bf16_bits(rng.standard_normal((2, 3, cfg.H, 512)).astype(np.float32))
    dout_f = bf16_bits_to_f32(dout).astype(np.float64)
    dq, dc = _run(hi, cfg, idx, dout, True)
    dq_ref, dc_ref = oracle.attend_bwd(hi.q[0], hi.c_kv[0], idx, hi.q_pos, 0, 0, 512, cfg.scale,
                                       dout_f)
    q = bf16_bits_to_f32(hi.q[0]).astype(np.float64)
    c = bf16_bits_to_f32(hi.c_kv[0]).astype(np.float64)
    m_dq = np.zeros_like(dq_ref)
    m_dc = np.zeros_like(dc_ref)
    for b in range(2):
        for i in range(3):
            keys = _keys_of(int(q_pos[b, i]), idx[b, i], 0, 0)
            assert len(keys) == min(2100, int(q_pos[b, i]) + 1)
            m_dq[b, i], rows = _row_bounds(q[b, i], c[b], keys, dout_f[b, i], cfg.scale, True)
            np.add.at(m_dc[b], keys, rows)
    _assert_grad_close(dq, dq_ref, m_dq, "dq")
    touched = m_dc.sum(axis=-1) > 0
    _assert_grad_close(dc[touched], dc_ref[touched], m_dc[touched], "dc")
    assert not dc[~touched].any()


def test_attend_bwd_empty_sets_and_bad_index():
    """No keys at all (sink = window = K_sparse = 0): dq is zero and dc untouched.  An index
    outside the dynamic region raises LSA_DEVERR_INDEX and its key is skipped, nothing faults."""
    cfg = LsaConfig("bwd_err", B=1, L=600, T=2, K=16 + 64 + 32, sink=16, swa=64, n_needles=0,
                    seed=51, H=32)
    hi = make_host_inputs(cfg, q_pos=np.array([[400, 599]], np.int32))
    q, c = dev_bf16(hi.q[0]), dev_bf16(hi.c_kv[0])
    kv, qp = dev_i32(hi.kv_len), dev_i32(hi.q_pos)
    dout = dev_bf16(to_bf16_bits(np.ones((1, 2, 32, 512), np.float32)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dc = lsa.lsa_attend_bwd(q, c, None, kv, qp, 0, 0, cfg.scale, dout, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and not bool(dq.any()) and not bool(dc.any())
    idx = oracle.index(hi.q_I, hi.w_I, hi.k_I, None, hi.kv_len, hi.q_pos, cfg.K_sparse, cfg.sink,
                       cfg.swa)
    idx[0, 1, 5] = 599  # inside the window, not the dynamic region
    lsa.lsa_attend_bwd(q, c, dev_i32(idx), kv, qp, cfg.sink, cfg.swa, cfg.scale, dout,
                       device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & lsa.DEVERR_INDEX


def test_attend_bwd_tc_empty_set_and_invalid_row():
    """The tcgen05 backward (64 heads, the forward's outputs): a query with no keys (sink =
    window = K_sparse = 0) gets dq = 0 and touches no row; a query position outside its sequence
    raises LSA_DEVERR_QPOS and gets dq = 0."""
    cfg = LsaConfig("bwd_tc_err", B=1, L=600, T=2, K=16, sink=0, swa=0, n_needles=0, seed=53,
                    H=64)
    hi = make_host_inputs(cfg, q_pos=np.array([[400, 599]], np.int32))
    q, c = dev_bf16(hi.q[0]), dev_bf16(hi.c_kv[0])
    kv, qp = dev_i32(hi.kv_len), dev_i32(hi.q_pos)
    idx = dev_i32(np.full((1, 2, 16), -1, np.int32))
    out, lse = lsa.lsa_attend(q, c, idx, kv, qp, 0, 0, cfg.scale)
    dout = dev_bf16(to_bf16_bits(np.ones((1, 2, 64, 512), np.float32)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dc = lsa.lsa_attend_bwd(q, c, idx, kv, qp, 0, 0, cfg.scale, dout, out=out, lse=lse,
                                device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and not bool(dq.any()) and not bool(dc.any())
    qp_bad = dev_i32(np.array([[400, 600]], np.int32))  # 600 = kv_len: outside
    dq, dc = lsa.lsa_attend_bwd(q, c, idx, kv, qp_bad, 16, 64, cfg.scale, dout, out=out,
                                lse=lse, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & lsa.DEVERR_QPOS
    assert not bool(dq[0, 1].any())


def test_attend_bwd_tc_bad_index_skipped():
    """The tcgen05 backward given an index inside the window (not the dynamic region) for one
    query: it raises LSA_DEVERR_INDEX, skips the bad slot (and any slot it leaves out of
    ascending order), keeps every output finite, and the other query's dq is bit-identical to
    the run on the clean index set."""
    cfg = LsaConfig("bwd_tc_idx", B=1, L=600, T=2, K=16 + 64 + 32, sink=16, swa=64, n_needles=0,
                    seed=57, H=64)
    hi = make_host_inputs(cfg, q_pos=np.array([[400, 599]], np.int32))
    q, c = dev_bf16(hi.q[0]), dev_bf16(hi.c_kv[0])
    kv, qp = dev_i32(hi.kv_len), dev_i32(hi.q_pos)
    idx = oracle.index(hi.q_I, hi.w_I, hi.k_I, None, hi.kv_len, hi.q_pos, cfg.K_sparse, cfg.sink,
                       cfg.swa)
    rng = np.random.default_rng(9)
    dout = dev_bf16(to_bf16_bits(rng.standard_normal((1, 2, 64, 512)).astype(np.float32)))
    bad = idx.copy()
    bad[0, 1, 5] = 599  # inside the window of t = 599
    out, lse = lsa.lsa_attend(q, c, dev_i32(idx), kv, qp, cfg.sink, cfg.swa, cfg.scale)
    res = []
    for rows in (idx, bad):
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        dq, dc = lsa.lsa_attend_bwd(q, c, dev_i32(rows), kv, qp, cfg.sink, cfg.swa, cfg.scale,
                                    dout, out=out, lse=lse, device_error=err)
        torch.cuda.synchronize()
        res.append((int(err.item()), dq.cpu().numpy(), dc.cpu().numpy()))
    assert res[0][0] == 0
    assert res[1][0] & lsa.DEVERR_INDEX
    assert np.isfinite(res[1][1]).all() and np.isfinite(res[1][2]).all()
    assert np.array_equal(res[0][1][0, 0], res[1][1][0, 0])
