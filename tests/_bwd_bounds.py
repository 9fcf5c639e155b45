"""Error bound of the HFA backward's parity tests (shared by the GPU tests and the CPU test that
checks the bound itself).  An element may differ from the fp64 oracle by
    1e-3 |ref| + 4e-3 R + 1e-5 M
  R: the size of the terms the kernel rounds to bf16 before the gradient products (relative
     error at most 2^-8 each): sum_s |scale dz_s| |c_s| for dq, and
     sum_h (|scale dz_hs| |q_h| + p_hs |dout_h|) for the row gradient of key s;
  M: the same sums with every factor in absolute value, dz_s replaced by
     p_s (|dout| |c_s| + |D| + |dp_s - D| |z_s|), which covers the fp32 sums, the cancellation
     in dp_s - D and the rounding of the exponent.
When the backward takes the forward's bf16 output and lse (D = dout . out), D carries the
forward's rounding of p and of out, at most E = 2^-7 sum_s p_s |dout| |c_s| per head, which
enters dz_s as p_s E scale: add scale E sum_s p_s |c_s| to dq and sum_h scale p_hs E_h |q_h| to
the row gradient of key s (with a 1.2 margin).
"""
import numpy as np

import oracle


def row_bounds(q, c_seq, keys, dout, scale, fwd_outputs=False):
    """Absolute bounds (4e-3 R + 1e-5 M, plus the forward's share when fwd_outputs) on the errors
    of dq [H, Dqk] and of the row gradients [len(keys), Dqk] of one query (q [H, Dqk],
    c_seq [L, Dqk], dout [H, Dv] as floats)."""
    C = c_seq[keys]
    z = scale * q @ C.T
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    dp = dout @ C[:, :512].T
    D = (p * dp).sum(axis=1, keepdims=True)
    rz = scale * p * np.abs(dp - D)
    r_dq = rz @ np.abs(C)
    r_dc = rz.T @ np.abs(q)
    r_dc[:, :512] += p.T @ np.abs(dout)
    wz = scale * p * (np.abs(dout) @ np.abs(C[:, :512]).T + np.abs(D) + np.abs(dp - D) * np.abs(z))
    m_dq = wz @ np.abs(C)
    m_dc = wz.T @ np.abs(q)
    m_dc[:, :512] += (p * (1.0 + np.abs(z))).T @ np.abs(dout)
    b_dq, b_dc = 4e-3 * r_dq + 1e-5 * m_dq, 4e-3 * r_dc + 1e-5 * m_dc
    if fwd_outputs:
        E = 2.0 ** -7 * (p * (np.abs(dout) @ np.abs(C[:, :512]).T)).sum(axis=1, keepdims=True)
        b_dq = b_dq + 1.2 * scale * E * (p @ np.abs(C))
        b_dc = b_dc + 1.2 * scale * (p * E).T @ np.abs(q)
    return b_dq, b_dc


def keys_of(t, idx_row, sink, swa):
    (s0, s1), (w0, w1), _ = oracle.regions(t, sink, swa)
    return np.concatenate([np.arange(s0, s1), np.arange(w0, w1),
                           idx_row[idx_row >= 0]]).astype(np.int64)


def error_report(got, ref, bound, what):
    """One line describing the error distribution against the oracle (printed by the tests, not
    gated): relative error in norm per row, and the element error over its tolerance."""
    got = np.asarray(got, np.float64).reshape(-1, np.shape(ref)[-1])
    ref = np.asarray(ref, np.float64).reshape(got.shape)
    bound = np.asarray(bound, np.float64).reshape(got.shape)
    norms = np.linalg.norm(ref, axis=1)
    # rows whose reference is (near) zero, e.g. a one-key query's dq, have no relative error
    live = norms > 1e-6 * max(float(norms.max()), 1e-30)
    rn = np.linalg.norm(got - ref, axis=1)[live] / norms[live] if live.any() else np.zeros(1)
    ratio = np.abs(got - ref) / (1e-3 * np.abs(ref) + bound)
    q = lambda x, p: float(np.percentile(x, p))
    return (f"{what}: row rel-err in norm p50 {q(rn, 50):.2e} p99 {q(rn, 99):.2e} max "
            f"{rn.max():.2e} ({int((~live).sum())} zero rows left out); err/tol p50 "
            f"{q(ratio, 50):.2e} p99.9 {q(ratio, 99.9):.2e} max {ratio.max():.2e}")


def assert_grad_close(got, ref, bound, what):
    print(error_report(got, ref, bound, what))
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    tol = 1e-3 * np.abs(ref) + bound
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance, worst err/tol "
                           f"{(err / tol).max():.3e}")
