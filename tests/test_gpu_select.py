"""Top-K selection at the edges of its two forms, through lsa_index.

Calls of at most 512 rows whose rows hold at most 16384 slots are selected in one launch per row;
others take the collect and final passes.  Both must give the oracle's selection (Sec. 2.2
Eq. 2: top K_sparse of dyn by score, ties to the lower position, output ascending) on the GPU's
own scores, bit-exact.  The keys repeat in groups, so runs of equal scores straddle the K-th
score and the tie rule decides part of the selection.  The first-digit threshold comes from the
tcgen05 scorer's fused histogram, or from the select's own histogram pass behind the CUDA-core
scorer.
"""
import numpy as np
import pytest

import oracle
from lightning_indexer_top_score_b200 import lsa
from lightning_indexer_top_score_b200.workloads import LsaConfig, make_host_inputs
from _tensors import dev_bf16, dev_i32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(params=["tcgen05", "legacy"])
def threshold_source(request, monkeypatch):
    """The threshold digit from the tcgen05 scorer, or from the select's own histogram pass
    (CUDA-core scorer)."""
    monkeypatch.delenv("LSA_NO_TCGEN05", raising=False)
    monkeypatch.delenv("LSA_SCORE_ONE_QUERY", raising=False)
    if request.param == "legacy":
        monkeypatch.setenv("LSA_NO_TCGEN05", "1")
    return request.param


def _grouped_keys(hi, group):
    """Every key row becomes the first row of its group of `group` consecutive positions."""
    B, L, _ = hi.k_I.shape
    src = (np.arange(L) // group) * group
    hi.k_I[:] = hi.k_I[:, src]


def _select_and_check(hi, cfg):
    B, T = hi.q_pos.shape
    L_max = hi.k_I.shape[1]
    q, w, k = dev_bf16(hi.q_I), dev_bf16(hi.w_I), dev_bf16(hi.k_I)
    dbg = torch.full((B, T, L_max), float("nan"), device="cuda")
    ws = torch.empty(lsa.lsa_index_workspace_bytes(B, T, cfg.H_I, cfg.D_I, L_max, cfg.K_sparse,
                                                   cfg.page, cfg.sub_block, 0),
                     dtype=torch.uint8, device="cuda")
    idx = lsa.lsa_index(q, w, k, None, dev_i32(hi.kv_len), dev_i32(hi.q_pos), cfg.K_sparse,
                        cfg.sink, cfg.swa, cfg.page, cfg.sub_block, 0, scores_dbg=dbg, ws=ws)
    assert lsa.lsa_get_error(ws) == 0
    idx, dbg = idx.cpu().numpy(), dbg.cpu().numpy()
    ties = 0
    for b in range(B):
        for i in range(T):
            t = int(hi.q_pos[b, i])
            want, m = oracle.select_query(dbg[b, i], None, t, cfg.K_sparse, cfg.sink, cfg.swa)
            assert idx[b, i].tolist() == want.tolist(), f"row ({b},{i}) t={t}"
            (_, _), (_, _), (lo, hi_) = oracle.regions(t, cfg.sink, cfg.swa)
            assert m == min(cfg.K_sparse, max(0, hi_ - lo))
            if m == cfg.K_sparse and m < hi_ - lo:
                # the K-th score is shared by a selected slot and one left out: the tie rule
                # (lower position first) decided between them
                kth = np.sort(dbg[b, i, lo:hi_])[::-1][m - 1]
                eq = lo + np.flatnonzero(dbg[b, i, lo:hi_] == kth)
                taken = np.isin(eq, want[:m])
                ties += int(taken.any() and not taken.all())
    return ties


@pytest.mark.parametrize("L", [16384, 16385])
def test_select_row_length_edge(L):
    """A 16384-token cache (rows of at most 16384 slots: the one-launch form) and a 16385-token
    one (collect + final)."""
    sink, swa = 16, 64
    cfg = LsaConfig("sel_len", B=2, L=L, T=2, H_I=64, K=sink + swa + 700, sink=sink, swa=swa,
                    n_needles=0, seed=61, H=8)
    hi = make_host_inputs(cfg, q_pos=np.array([[L - 1, L - 2], [L - 1, L // 2]], np.int32),
                          with_attention=False)
    _grouped_keys(hi, 7)
    ties = _select_and_check(hi, cfg)
    assert ties > 0, "no row had a tie across its K-th score"


@pytest.mark.parametrize("B", [512, 513])
def test_select_row_count_edge(B):
    """512 rows per call (one-launch form) and 513 (collect + final), short ragged rows."""
    sink, swa = 16, 64
    cfg = LsaConfig("sel_rows", B=B, L=900, T=1, H_I=64, K=sink + swa + 120, sink=sink,
                    swa=swa, n_needles=0, seed=67, H=8)
    rng = np.random.default_rng(3)
    kv_len = rng.integers(60, 901, size=B).astype(np.int32)
    hi = make_host_inputs(cfg, kv_len=kv_len, with_attention=False)
    _grouped_keys(hi, 5)
    ties = _select_and_check(hi, cfg)
    assert ties > 0, "no row had a tie across its K-th score"


@pytest.mark.parametrize("L", [16500, 131073])
def test_select_unaligned_rows(L, threshold_source):
    """Collect + final on rows whose dyn region starts off a 16-byte boundary (an odd sink: a
    scalar head and a ragged tail around the float4 body of each chunk)."""
    sink, swa = 5, 100
    cfg = LsaConfig("sel_unaligned", B=2, L=L, T=2, H_I=64, K=sink + swa + 2048, sink=sink,
                    swa=swa, n_needles=0, seed=71, H=8)
    hi = make_host_inputs(cfg, q_pos=np.array([[L - 1, L - 3], [L - 2, L // 3]], np.int32),
                          with_attention=False)
    _grouped_keys(hi, 11)
    ties = _select_and_check(hi, cfg)
    assert ties > 0, "no row had a tie across its K-th score"


def test_select_all_scores_equal(threshold_source):
    """Every key the same, so every dyn score of a row is equal: the whole dyn region (more than
    the 8192 candidates the final pass keeps in shared memory) is the candidate list, read back
    from the global list, and the lowest positions win."""
    sink, swa = 16, 64
    L = 30000
    cfg = LsaConfig("sel_equal", B=2, L=L, T=2, H_I=64, K=sink + swa + 1500, sink=sink,
                    swa=swa, n_needles=0, seed=79, H=8)
    hi = make_host_inputs(cfg, q_pos=np.array([[L - 1, 20000], [L - 7, 9000]], np.int32),
                          with_attention=False)
    hi.k_I[:] = hi.k_I[:, :1]
    _select_and_check(hi, cfg)
