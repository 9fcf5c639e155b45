"""HFA backward (lsa_attend_bwd) through the C-ABI against the fp64 oracle.

The index sets come from the oracle's own indexer on the same host inputs.  Tolerance, from the
arithmetic: every sum is fp32 over products of bf16-exact values, plus exp2f and the fp32 online
lse / D.  Where attention is flat over identical rows (the planted needles repeat one row), dp_s - D
cancels to rounding, so the bound on an element is relative to the size of the terms that form it,
not to the result: |got - ref| <= 1e-3 |ref| + 1e-5 M, where M is the same expression with every
term in absolute value (dz_s replaced by p_s (|dout||c_s| + |D| + |dp_s - D||z_s|), the last part
covering the rounding of the exponent).  A dropped term, a wrong sign or a wrong row moves an
element by a sizeable share of M.
"""
import numpy as np
import pytest

import oracle
from lightning_indexer_top_score_b200 import lsa
from lightning_indexer_top_score_b200.workloads import (LsaConfig, bf16_bits_to_f32,
                                                        make_host_inputs, to_bf16_bits)
from _tensors import dev_bf16, dev_i32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _row_bounds(q, c_seq, keys, dout, scale):
    """fp64 sizes M of the terms of dq [H, Dqk] and of the row gradients [len(keys), Dqk] of one
    query (q [H, Dqk], c_seq [L, Dqk], dout [H, Dv] as floats)."""
    C = c_seq[keys]
    z = scale * q @ C.T
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    dp = dout @ C[:, :512].T
    D = (p * dp).sum(axis=1, keepdims=True)
    wz = scale * p * (np.abs(dout) @ np.abs(C[:, :512]).T + np.abs(D) + np.abs(dp - D) * np.abs(z))
    m_dq = scale * wz @ np.abs(C)
    m_dc = scale * wz.T @ np.abs(q)
    m_dc[:, :512] += (p * (1.0 + np.abs(z))).T @ np.abs(dout)
    return m_dq, m_dc


def _keys_of(t, idx_row, sink, swa):
    (s0, s1), (w0, w1), _ = oracle.regions(t, sink, swa)
    return np.concatenate([np.arange(s0, s1), np.arange(w0, w1),
                           idx_row[idx_row >= 0]]).astype(np.int64)


def _assert_grad_close(got, ref, mag, what):
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    tol = 1e-3 * np.abs(ref) + 1e-5 * mag
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance, worst err/tol "
                           f"{(err / tol).max():.3e}")


def _run(hi, cfg, idx, dout_bits):
    q, c = dev_bf16(hi.q[0]), dev_bf16(hi.c_kv[0])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dc = lsa.lsa_attend_bwd(q, c, dev_i32(idx), dev_i32(hi.kv_len), dev_i32(hi.q_pos),
                                cfg.sink, cfg.swa, cfg.scale, dev_bf16(dout_bits),
                                device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return dq.cpu().numpy(), dc.cpu().numpy()


def test_attend_bwd_ragged_shared_rows():
    """Three sequences in a larger cache, six queries each (window rows shared between queries,
    so their gradients accumulate; t = 0 has one key), 16 heads."""
    cfg = LsaConfig("bwd", B=3, L=1300, T=6, K=16 + 256 + 100, sink=16, swa=256, n_needles=4,
                    L_max=1400, seed=41, H=16)
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
    dq, dc = _run(hi, cfg, idx, dout)
    dq_ref, dc_ref = oracle.attend_bwd(hi.q[0], hi.c_kv[0], idx, hi.q_pos, cfg.sink, cfg.swa, 512,
                                       cfg.scale, dout_f)
    q = bf16_bits_to_f32(hi.q[0]).astype(np.float64)
    c = bf16_bits_to_f32(hi.c_kv[0]).astype(np.float64)
    m_dq = np.zeros_like(dq_ref)
    m_dc = np.zeros_like(dc_ref)
    for b in range(3):
        for i in range(6):
            keys = _keys_of(int(q_pos[b, i]), idx[b, i], cfg.sink, cfg.swa)
            m_dq[b, i], rows = _row_bounds(q[b, i], c[b], keys, dout_f[b, i], cfg.scale)
            np.add.at(m_dc[b], keys, rows)
    assert not dq[0, 0].any() and not dq_ref[0, 0].any()  # one key: p = 1, dz = 0
    _assert_grad_close(dq, dq_ref, m_dq, "dq")
    touched = m_dc.sum(axis=-1) > 0
    _assert_grad_close(dc[touched], dc_ref[touched], m_dc[touched], "dc (rows of some S_t)")
    assert not dc[~touched].any(), "gradient written to a row outside every S_t"


def test_attend_bwd_decode_128_heads_sampled():
    """128 heads (8 head groups per query), 4 sequences of 16384 tokens, one query each, K = 2048
    (16 + 1024 + 1008); two sequences checked in full (dq and every row gradient)."""
    cfg = LsaConfig("bwd_decode", B=4, L=16384, T=1, n_needles=8, seed=43)
    hi = make_host_inputs(cfg)
    idx = oracle.index(hi.q_I, hi.w_I, hi.k_I, None, hi.kv_len, hi.q_pos, cfg.K_sparse, cfg.sink,
                       cfg.swa)
    rng = np.random.default_rng(6)
    dout = to_bf16_bits(rng.standard_normal((4, 1, cfg.H, 512)).astype(np.float32))
    dq, dc = _run(hi, cfg, idx, dout)
    for b in (0, 3):
        t = int(hi.q_pos[b, 0])
        dout_f = bf16_bits_to_f32(dout[b, 0]).astype(np.float64)
        dq_ref, dc_ref = oracle.attend_bwd_query(hi.q[0][b, 0], hi.c_kv[0][b], idx[b, 0], t,
                                                 cfg.sink, cfg.swa, 512, cfg.scale, dout_f)
        keys = _keys_of(t, idx[b, 0], cfg.sink, cfg.swa)
        assert len(keys) == 2048
        m_dq, rows = _row_bounds(bf16_bits_to_f32(hi.q[0][b, 0]).astype(np.float64),
                                 bf16_bits_to_f32(hi.c_kv[0][b]).astype(np.float64), keys, dout_f,
                                 cfg.scale)
        _assert_grad_close(dq[b, 0], dq_ref, m_dq, f"dq sequence {b}")
        _assert_grad_close(dc[b][keys], dc_ref[keys], rows, f"dc sequence {b}")
        others = np.ones(dc.shape[1], bool)
        others[keys] = False
        assert not dc[b][others].any()
