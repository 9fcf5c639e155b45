"""Checks of the Hierarchical Indexing stage-2 token scores (LongCat Sparse Attention, Sec. 3.3
Eq. 10-11) shared by the small and the full-size GPU tests.

Stage 2 scores Eq. 1 on every token of the recalled pages that lies in the query's dynamic region,
and on nothing else.  The recalled pages are the top M of the stage-1 page scores by (score desc,
page asc) over the pages that intersect dyn; the oracle picks them here from the GPU's own page
scores, so the scored set is compared exactly and each scored value against fp64 Eq. 1."""
import numpy as np

import oracle
from _tensors import assert_scores_close, score_tolerance


def recalled_domain(page_row, t, sink, swa, page, M):
    """(recalled page ids ascending, their tokens within dyn ascending) as the oracle selects
    them from the fp32 page scores `page_row` (indexed by absolute page id)."""
    (_, _), (_, _), (lo, hi) = oracle.regions(t, sink, swa)
    if hi <= lo:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    pages = np.arange(lo // page, (hi - 1) // page + 1, dtype=np.int64)
    rec, m = oracle.topk(page_row[pages].astype(np.float64), pages, M)
    rec = rec[:m].astype(np.int64)
    toks = (rec[:, None] * page + np.arange(page)[None, :]).reshape(-1)
    toks = toks[(toks >= lo) & (toks < hi)]
    return rec, toks


def check_stage2_row(tok_row, page_row, q, w, k_seq, t, sink, swa, page, M, what,
                     sample=None, rng=None):
    """tok_row: the GPU's stage-2 scores at absolute positions (NaN where nothing was written);
    k_seq: the sequence's key cache [L, D] as bf16 bits, or a function returning the bf16 bits
    of the key rows at given positions (for caches that stay on the device)."""
    rec, dom = recalled_domain(page_row, t, sink, swa, page, M)
    scored = np.nonzero(~np.isnan(tok_row))[0]
    assert np.array_equal(scored, dom), (
        f"{what}: scored set differs from the recalled pages within dyn "
        f"({len(scored)} scored, {len(dom)} expected, "
        f"{len(np.setxor1d(scored, dom))} differ)")
    chk = dom
    if sample is not None and len(dom) > sample:
        chk = np.sort(rng.choice(dom, sample, replace=False))
    if len(chk):
        rows = k_seq(chk) if callable(k_seq) else np.asarray(k_seq)[chk]
        ref = oracle.scores(q, w, rows, np.arange(len(chk)))
        tol = score_tolerance(q, w, rows, ref)
        assert_scores_close(tok_row[chk], ref, tol, f"{what}: stage-2 scores")
    return rec, dom
