"""FP8 (E4M3) indexer through the C-ABI against the oracle.

The quantiser's codes must equal the oracle's codes of the same bf16 rows, and its scales must
match bit for bit.  Scores are then compared with the oracle's Eq. 1 on its own decoded codes,
within an fp32-accumulation tolerance.  Index sets must be bit-exact: the oracle selects from
the GPU's own fp32 scores.
"""
import numpy as np
import pytest

import oracle
from lightning_indexer_top_score_b200 import lsa
from lightning_indexer_top_score_b200.workloads import (DECODE_128K, DeviceInputs, LsaConfig,
                                                        make_host_inputs, to_bf16_bits)
from _tensors import assert_scores_close, dev_bf16, dev_i32, host_bits

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

_E4M3 = np.array([oracle.e4m3_value(c) for c in range(256)])  # NaN codes never appear


def _values(codes):
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def _quant_dev(x_dev):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales = lsa.lsa_quantize_fp8(x_dev, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return codes, scales


def _assert_same_quantisation(codes_dev, scales_dev, x_bits, what):
    c_ref, s_ref = oracle.quantize_e4m3(x_bits)
    np.testing.assert_array_equal(scales_dev.cpu().numpy(), s_ref, err_msg=f"{what} scales")
    np.testing.assert_array_equal(_values(codes_dev.cpu().numpy()), _values(c_ref),
                                  err_msg=f"{what} codes")
    return c_ref, s_ref


def _fp8_tolerance(q8, qs, w, k8, ks, ref):
    """fp32 accumulation of exact E4M3 products: 1e-3 relative plus 1e-5 of the magnitude sum."""
    wf = np.abs(oracle_w(w))
    mag = np.abs(_values(k8)) @ np.abs(_values(q8)).T * qs[None, :] * ks[:, None]
    return 1e-3 * np.abs(ref) + 1e-5 * (mag @ wf) + 1e-30


def oracle_w(w_bits):
    from lightning_indexer_top_score_b200.workloads import bf16_bits_to_f32
    return bf16_bits_to_f32(w_bits).astype(np.float64)


def test_quantize_matches_oracle():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((300, 128)).astype(np.float32)
    x *= (10.0 ** rng.uniform(-6, 4, 300)).astype(np.float32)[:, None]
    x[7] = 0.0
    x[11, :] = 1e-30            # flushes to bf16 subnormals / zero
    x[13, 5] = -4000.0          # one large element: the rest lands in the subnormal codes
    xb = to_bf16_bits(x)
    codes, scales = _quant_dev(dev_bf16(xb))
    _assert_same_quantisation(codes, scales, xb, "random rows")
    assert scales[7].item() == 0.0 and not codes[7].any().item()


def test_quantize_flags_nonfinite_input():
    x = np.ones((4, 64), np.float32)
    x[2, 3] = np.inf
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_quantize_fp8(dev_bf16(to_bf16_bits(x)), device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & 0x2


@pytest.mark.parametrize("H_I", [64, 128])
def test_index_fp8_ragged(H_I):
    """Three sequences of different lengths in a larger cache, six queries each at boundary
    positions (empty dyn, one-token dyn, mid, last)."""
    cfg = LsaConfig("fp8", B=3, L=1300, T=6, H_I=H_I, K=16 + 256 + 100, sink=16, swa=256,
                    n_needles=4, L_max=1400, seed=31, H=16)
    kv_len = np.array([1000, 517, 1300], np.int32)
    q_pos = np.array([[0, 10, 271, 272, 600, 999],
                      [516, 300, 15, 16, 290, 500],
                      [1299, 1298, 1000, 273, 700, 1200]], np.int32)
    hi = make_host_inputs(cfg, q_pos=q_pos, kv_len=kv_len)
    B, T, L_max = 3, 6, hi.k_I.shape[1]
    q8, qs = _quant_dev(dev_bf16(hi.q_I))
    k8, ks = _quant_dev(dev_bf16(hi.k_I))
    q8_ref, qs_ref = _assert_same_quantisation(q8, qs, hi.q_I, "queries")
    k8_ref, ks_ref = _assert_same_quantisation(k8, ks, hi.k_I, "keys")
    dbg = torch.full((B, T, L_max), float("nan"), device="cuda")
    ws = torch.empty(lsa.lsa_index_workspace_bytes(B, T, H_I, 128, L_max, cfg.K_sparse, 128, 8, 0),
                     dtype=torch.uint8, device="cuda")
    idx = lsa.lsa_index_fp8(q8, qs, dev_bf16(hi.w_I), k8, ks, dev_i32(hi.kv_len),
                            dev_i32(hi.q_pos), cfg.K_sparse, cfg.sink, cfg.swa, scores_dbg=dbg,
                            ws=ws)
    assert lsa.lsa_get_error(ws) == 0
    idx, dbg = idx.cpu().numpy(), dbg.cpu().numpy()
    for b in range(B):
        for i in range(T):
            t = int(hi.q_pos[b, i])
            (_, _), (_, _), (lo, hi_) = oracle.regions(t, cfg.sink, cfg.swa)
            dom = np.arange(lo, hi_)
            if len(dom):
                ref = oracle.scores_fp8(q8_ref[b, i], qs_ref[b, i], hi.w_I[b, i], k8_ref[b],
                                        ks_ref[b], dom)
                tol = _fp8_tolerance(q8_ref[b, i], qs_ref[b, i], hi.w_I[b, i], k8_ref[b][dom],
                                     ks_ref[b][dom], ref)
                assert_scores_close(dbg[b, i, dom], ref, tol, f"row ({b},{i}) t={t}")
            want, m = oracle.select_query(dbg[b, i], None, t, cfg.K_sparse, cfg.sink, cfg.swa)
            assert idx[b, i].tolist() == want.tolist(), f"indices row ({b},{i}) t={t}"
            assert m == min(cfg.K_sparse, max(0, hi_ - lo))


def test_index_fp8_decode_128k_sampled():
    """The decode workload at its full size (32 x 131072 keys): sampled rows' codes and scores,
    and exact selection for two sequences."""
    cfg = DECODE_128K
    inp = DeviceInputs(cfg, with_attention=False)
    k8, ks = _quant_dev(inp.k_I)
    q8, qs = _quant_dev(inp.q_I)
    B, T, L = cfg.B, cfg.T, cfg.L
    dbg = torch.full((B, T, L), float("nan"), device="cuda")
    idx = lsa.lsa_index_fp8(q8, qs, inp.w_I, k8, ks, inp.kv_len, inp.q_pos, cfg.K_sparse,
                            cfg.sink, cfg.swa, scores_dbg=dbg)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    rng = np.random.default_rng(4)
    for b in (0, 31):
        t = int(inp.q_pos[b, 0].item())
        (_, _), (_, _), (lo, hi) = oracle.regions(t, cfg.sink, cfg.swa)
        pos = np.sort(rng.choice(np.arange(lo, hi), 2048, replace=False)).astype(np.int64)
        kb = host_bits(inp.k_I[b, torch.from_numpy(pos).cuda()])
        k8_ref, ks_ref = _assert_same_quantisation(k8[b, torch.from_numpy(pos).cuda()],
                                                   ks[b, torch.from_numpy(pos).cuda()], kb,
                                                   f"keys of sequence {b}")
        qb = host_bits(inp.q_I[b, 0])
        q8_ref, qs_ref = _assert_same_quantisation(q8[b, 0], qs[b, 0], qb, f"query {b}")
        w = host_bits(inp.w_I[b, 0])
        ref = oracle.scores_fp8(q8_ref, qs_ref, w, k8_ref, ks_ref, np.arange(len(pos)))
        row = dbg[b, 0].cpu().numpy()
        assert_scores_close(row[pos], ref, _fp8_tolerance(q8_ref, qs_ref, w, k8_ref, ks_ref, ref),
                            f"sequence {b}")
        want, _ = oracle.select_query(row, None, t, cfg.K_sparse, cfg.sink, cfg.swa)
        assert idx[b, 0].tolist() == want.tolist(), f"indices sequence {b}"


def test_quantize_into_cache_slots():
    """Strided output: one token's key of every sequence written into its slot of a
    [B, L_max, D] FP8 cache equals the contiguous quantisation, and no other slot changes."""
    rng = np.random.default_rng(9)
    keys = to_bf16_bits(rng.standard_normal((3, 128)).astype(np.float32))
    k8 = torch.full((3, 10, 128), 0x55, dtype=torch.uint8, device="cuda")
    ks = torch.full((3, 10), -1.0, dtype=torch.float32, device="cuda")
    lsa.lsa_quantize_fp8(dev_bf16(keys), codes=k8[:, 5], scales=ks[:, 5])
    c_ref, s_ref = _quant_dev(dev_bf16(keys))
    assert torch.equal(k8[:, 5], c_ref) and torch.equal(ks[:, 5], s_ref)
    others = [j for j in range(10) if j != 5]
    assert bool((k8[:, others] == 0x55).all()) and bool((ks[:, others] == -1.0).all())
