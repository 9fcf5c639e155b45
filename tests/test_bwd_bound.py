"""The HFA backward's parity bound admits the kernel's bf16 rounding of p and dz but rejects
plausible mistakes.  Each variant below is the gradient computed in numpy from the same inputs
(a restatement used only to exercise the bound; the oracle is pinned elsewhere):
  - p and dz rounded to bf16 before the products, as the kernel does: must pass;
  - D taken from the forward's bf16 output (the fast path), under the bound with the
    forward's share: must pass;
  - D dropped from dz, the p dout term of dc with its sign flipped, and row gradients written
    one row off: each must fail (a dropped D under both bounds)."""
import numpy as np
import pytest

import oracle
from lightning_indexer_top_score_b200.workloads import (LsaConfig, bf16_bits_to_f32,
                                                        make_host_inputs, to_bf16_bits)
from _bwd_bounds import keys_of, row_bounds


def _bf16(x):
    return bf16_bits_to_f32(to_bf16_bits(np.asarray(x, np.float32))).astype(np.float64)


def _grads(q, C, dout, scale, round_bf16=False, drop_D=False, flip_pdout=False,
           D_from_bf16_out=False):
    z = scale * q @ C.T
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    dp = dout @ C[:, :512].T
    D = 0.0 if drop_D else (p * dp).sum(axis=1, keepdims=True)
    if D_from_bf16_out:
        # the forward's output after its two roundings (p, then out), as the fast path reads it
        out = _bf16(_bf16(p) @ C[:, :512])
        D = (dout * out).sum(axis=1, keepdims=True)
    dzs = p * (dp - D) * scale
    if round_bf16:
        p, dzs = _bf16(p), _bf16(dzs)
    dq = dzs @ C
    dc = dzs.T @ q
    dc[:, :512] += (-1.0 if flip_pdout else 1.0) * (p.T @ dout)
    return dq, dc


def _fails(got, ref, bound):
    return bool((np.abs(got - ref) > 1e-3 * np.abs(ref) + bound).any())


@pytest.fixture(scope="module")
def case():
    cfg = LsaConfig("bound", B=1, L=700, T=1, K=16 + 128 + 96, sink=16, swa=128, n_needles=4,
                    seed=17, H=32)
    hi = make_host_inputs(cfg, q_pos=np.array([[650]], np.int32))
    idx = oracle.index(hi.q_I, hi.w_I, hi.k_I, None, hi.kv_len, hi.q_pos, cfg.K_sparse, cfg.sink,
                       cfg.swa)
    rng = np.random.default_rng(3)
    dout = _bf16(rng.standard_normal((cfg.H, 512)))
    t = 650
    keys = keys_of(t, idx[0, 0], cfg.sink, cfg.swa)
    q = bf16_bits_to_f32(hi.q[0][0, 0]).astype(np.float64)
    c = bf16_bits_to_f32(hi.c_kv[0][0]).astype(np.float64)
    dq_ref, dc_ref = oracle.attend_bwd_query(hi.q[0][0, 0], hi.c_kv[0][0], idx[0, 0], t, cfg.sink,
                                             cfg.swa, 512, cfg.scale, dout)
    m_dq, m_dc = row_bounds(q, c, keys, dout, cfg.scale)
    f_dq, f_dc = row_bounds(q, c, keys, dout, cfg.scale, fwd_outputs=True)
    return dict(q=q, C=c[keys], dout=dout, scale=cfg.scale, dq=dq_ref, dc=dc_ref[keys],
                m_dq=m_dq, m_dc=m_dc, f_dq=f_dq, f_dc=f_dc)


def test_bound_admits_bf16_operands(case):
    dq, dc = _grads(case["q"], case["C"], case["dout"], case["scale"], round_bf16=True)
    assert not _fails(dq, case["dq"], case["m_dq"])
    assert not _fails(dc, case["dc"], case["m_dc"])


def test_bound_rejects_dropped_D(case):
    dq, _ = _grads(case["q"], case["C"], case["dout"], case["scale"], drop_D=True)
    assert _fails(dq, case["dq"], case["m_dq"])


def test_bound_rejects_flipped_p_dout(case):
    _, dc = _grads(case["q"], case["C"], case["dout"], case["scale"], flip_pdout=True)
    assert _fails(dc, case["dc"], case["m_dc"])


def test_bound_rejects_rows_one_off(case):
    _, dc = _grads(case["q"], case["C"], case["dout"], case["scale"])
    assert not _fails(dc, case["dc"], case["m_dc"])
    assert _fails(np.roll(dc, 1, axis=0), case["dc"], case["m_dc"])


def test_bound_with_forward_outputs(case):
    dq, dc = _grads(case["q"], case["C"], case["dout"], case["scale"], round_bf16=True,
                    D_from_bf16_out=True)
    assert not _fails(dq, case["dq"], case["f_dq"])
    assert not _fails(dc, case["dc"], case["f_dc"])
    dq, dc = _grads(case["q"], case["C"], case["dout"], case["scale"], drop_D=True)
    assert _fails(dq, case["dq"], case["f_dq"]) and _fails(dc, case["dc"], case["f_dc"])
