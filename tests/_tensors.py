"""Host <-> device conversion helpers for the tests (bf16 bit patterns <-> torch.bfloat16),
and the tolerance formulas the parity tests apply."""
import numpy as np


def dev_bf16(bits: np.ndarray, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def host_bits(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def dev_i32(a, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def bf16_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def score_tolerance(q_bits, w_bits, k_bits, ref):
    """|I_gpu - I_64| <= 1e-3 |I_64| + 1e-5 * sum_j |w_j| sum_d |q_jd k_d|  (per element).
    q [H,D], w [H], k [n,D], ref [n]."""
    q, w, k = bf16_f64(q_bits), bf16_f64(w_bits), bf16_f64(k_bits)
    mag = np.abs(k) @ (np.abs(w) @ np.abs(q))
    return 1e-3 * np.abs(ref) + 1e-5 * mag


def assert_scores_close(got, ref, tol, what=""):
    err = np.abs(np.asarray(got, np.float64) - ref)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, (f"{what}: {bad.size} scores out of tolerance; worst "
                           f"{err.max():.3e} at {int(np.argmax(err))}")


def assert_attention_close(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    """bf16 output: |d| <= 1e-2 + 2e-2 |ref|; lse within 1e-3 absolute."""
    o = np.asarray(out_gpu, np.float64)
    err = np.abs(o - out_ref)
    lim = 1e-2 + 2e-2 * np.abs(out_ref)
    assert np.all(err <= lim), f"{what}: out worst |d| {err.max():.3e}"
    le = np.abs(np.asarray(lse_gpu, np.float64) - lse_ref)
    assert np.all(le <= 1e-3), f"{what}: lse worst |d| {le.max():.3e}"
