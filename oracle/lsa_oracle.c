/*
 * lsa_oracle.c -- plain, slow, fp64 CPU oracle for the LongCat Sparse Attention
 * (LSA) layer hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library; the two meet only through the bytes of the seeded inputs.
 *
 * Source: "LongCat Sparse Attention: Taming the Lightning via Streaming-aware
 * Hierarchical Cross-Layer Indexing" (arXiv 2608.01662).  Each function names
 * the section / equation it restates.  Index conventions are 0-based: query
 * position t attends key positions 0..t.
 *
 * Precision: bf16 inputs are widened exactly to double; every sum is a plain
 * sequential fp64 sum.  No blocking, fusion or reordering beyond what the
 * equations state.  Sorting uses the C library qsort.
 *
 * Readings where the pages are silent (all listed again in the design notes):
 *  - region split: sink = [0, min(Ks, t+1)), swa = [max(Ks, t-Kw+1), t],
 *    dyn = [Ks, t-Kw]; the three sets are disjoint (Sec. 3.1, budget split).
 *  - ties in every arg-top-K break toward the lower position / page id; the
 *    selected set is returned sorted ascending and padded with -1.
 *  - HI: only pages that intersect dyn are ranked; the token domain of stage 2
 *    is (recalled pages) intersected with dyn (Sec. 3.3, Eq. 9-11 with SI).
 *  - a sub-block mean is the mean of the tokens present (a partial last block
 *    averages fewer tokens).
 *  - attention: natural-log LSE, V = first Dv dims of the latent row.
 *  - MinMax pooling (Sec. 5.3.5 gives only the sub-block term): the term takes
 *    the place of q . k_mean inside Eq. 9, ReLU and head weights unchanged.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- helpers */

static double bf(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------ a1: region split
 * Streaming-aware Indexing (Sec. 3.1, budget partition S_t = S_sink U S_swa U
 * S_sparse, mutually exclusive).  The pages write S_sink = {1..K_sink} and
 * S_swa = {t-K_swa+1..t} 1-based; here 0-based, clipped to be disjoint and
 * causal.  Output r[6] = half-open [sink_lo, sink_hi), [swa_lo, swa_hi),
 * [dyn_lo, dyn_hi).  With Ks = Kw = 0 (plain DSA) dyn = [0, t].
 */
void orc_regions(int64_t t, int Ks, int Kw, int64_t r[6])
{
    int64_t sink_hi = (t + 1 < Ks) ? t + 1 : Ks;
    int64_t swa_lo = t - Kw + 1;
    if (swa_lo < Ks) swa_lo = Ks;
    int64_t swa_hi = t + 1;
    if (swa_hi < swa_lo) swa_hi = swa_lo;
    int64_t dyn_lo = Ks;
    int64_t dyn_hi = t - Kw + 1;
    if (dyn_hi < dyn_lo) dyn_hi = dyn_lo;
    r[0] = 0;
    r[1] = sink_hi;
    r[2] = swa_lo;
    r[3] = swa_hi;
    r[4] = dyn_lo;
    r[5] = dyn_hi;
}

/* ------------------------------------------------- a2: indexer score Eq.1
 * I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s])   (Sec. 2.2, Eq. 1)
 * q: [H*D] bf16 of one query, w: [H] bf16, key: [D] bf16.
 */
double orc_score_one(const uint16_t *q, const uint16_t *w, const uint16_t *key,
                     int H, int D)
{
    double I = 0.0;
    for (int j = 0; j < H; ++j) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf(q[(int64_t)j * D + d]) * bf(key[d]);
        if (dot > 0.0) I += bf(w[j]) * dot;
    }
    return I;
}

/* Scores of one query against keys at the given positions of one sequence. */
void orc_scores(const uint16_t *q, const uint16_t *w, const uint16_t *k_seq,
                int H, int D, const int64_t *pos, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_score_one(q, w, k_seq + pos[i] * D, H, D);
}

/* ------------------------------------------------ a3: arg-top-K (Eq. 2)
 * S = arg topK over the candidates, ranked by (score desc, position asc).
 * Returns the number selected m = min(K, n); out[0..m) holds the selected
 * positions sorted ascending, out[m..K) = -1.
 */
typedef struct { double s; int64_t p; } cand_t;

static int cmp_rank(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->p < y->p) ? -1 : (x->p > y->p);
}

static int cmp_i64(const void *a, const void *b)
{
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x < y) ? -1 : (x > y);
}

int64_t orc_topk(const double *score, const int64_t *pos, int64_t n, int K,
                 int32_t *out)
{
    int64_t m = n < K ? n : K;
    if (m < 0) m = 0;
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
    int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * (size_t)(m > 0 ? m : 1));
    for (int64_t i = 0; i < n; ++i) { c[i].s = score[i]; c[i].p = pos[i]; }
    qsort(c, (size_t)n, sizeof(cand_t), cmp_rank);
    for (int64_t i = 0; i < m; ++i) sel[i] = c[i].p;
    qsort(sel, (size_t)m, sizeof(int64_t), cmp_i64);
    for (int64_t i = 0; i < K; ++i) out[i] = (i < m) ? (int32_t)sel[i] : -1;
    free(c);
    free(sel);
    return m;
}

/* --------------------------------------------- a4: sub-block mean cache
 * k_mean[n] = mean of k over sub-block n = [n*B, (n+1)*B) intersected with
 * [0, L)  (Sec. 3.3: Hierarchical Indexing reads these means from a
 * per-sequence cache, not from the keys at query time).  out: [ceil(L/B) * D] doubles.
 */
void orc_block_means(const uint16_t *k_seq, int64_t L, int D, int B, double *out)
{
    int64_t nb = (L + B - 1) / B;
    for (int64_t n = 0; n < nb; ++n) {
        int64_t lo = n * B, hi = lo + B < L ? lo + B : L;
        for (int d = 0; d < D; ++d) {
            double s = 0.0;
            for (int64_t i = lo; i < hi; ++i) s += bf(k_seq[i * D + d]);
            out[n * D + d] = s / (double)(hi - lo);
        }
    }
}

/* ------------------------------------------------- a5: page score Eq. 9
 * I_page[t,p] = sum_j w[t,j] * sum_{n in page p} ReLU(q[t,j] . k_mean[n])
 * k_mean: the stored bf16 sub-block means of one sequence ([ceil(L/B)*D]).
 * Sub-blocks of page p are n = p*P/B .. (p+1)*P/B - 1 that exist for length L.
 */
double orc_page_score(const uint16_t *q, const uint16_t *w, const uint16_t *kmean_seq,
                      int H, int D, int64_t L, int P, int B, int64_t p)
{
    int64_t nb = (L + B - 1) / B;
    int64_t n_lo = p * (P / B), n_hi = n_lo + P / B;
    if (n_hi > nb) n_hi = nb;
    double I = 0.0;
    for (int j = 0; j < H; ++j) {
        double inner = 0.0;
        for (int64_t n = n_lo; n < n_hi; ++n) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += bf(q[(int64_t)j * D + d]) * bf(kmean_seq[n * D + d]);
            if (dot > 0.0) inner += dot;
        }
        I += bf(w[j]) * inner;
    }
    return I;
}

/* ------------------------- f4: MinMax sub-block pooling (Sec. 5.3.5)
 * The pooling ablation of Sec. 5.3.5 (Table 11) keeps, instead of the mean
 * key of sub-block n, its element-wise extremes over the tokens present:
 *   k_max[n,d] = max_{s in n} k[s,d],   k_min[n,d] = min_{s in n} k[s,d].
 * Both are values of the bf16 cache, so they are exact.
 * out: [ceil(L/B) * 2D] doubles, row n = (k_max[n, 0..D), k_min[n, 0..D)).
 */
void orc_block_minmax(const uint16_t *k_seq, int64_t L, int D, int B, double *out)
{
    int64_t nb = (L + B - 1) / B;
    for (int64_t n = 0; n < nb; ++n) {
        int64_t lo = n * B, hi = lo + B < L ? lo + B : L;
        for (int d = 0; d < D; ++d) {
            double mx = bf(k_seq[lo * D + d]), mn = mx;
            for (int64_t i = lo + 1; i < hi; ++i) {
                double v = bf(k_seq[i * D + d]);
                if (v > mx) mx = v;
                if (v < mn) mn = v;
            }
            out[n * 2 * D + d] = mx;
            out[n * 2 * D + D + d] = mn;
        }
    }
}

/* Page score with MinMax pooling.  Sec. 5.3.5 defines the sub-block term
 *   s~[t,n,j] = sum_d max(q[t,j,d] * k_max[n,d], q[t,j,d] * k_min[n,d]);
 * the reading here puts it in place of q[t,j] . k_mean[n] in Eq. 9:
 *   I_page[t,p] = sum_j w[t,j] * sum_{n in page p} ReLU(s~[t,n,j]).
 * kmm_seq: the stored rows of one sequence, [ceil(L/B) * 2D] bf16 bits, row n
 * = (k_max[n], k_min[n]).  Sub-blocks as in orc_page_score.
 */
double orc_page_score_minmax(const uint16_t *q, const uint16_t *w, const uint16_t *kmm_seq,
                             int H, int D, int64_t L, int P, int B, int64_t p)
{
    int64_t nb = (L + B - 1) / B;
    int64_t n_lo = p * (P / B), n_hi = n_lo + P / B;
    if (n_hi > nb) n_hi = nb;
    double I = 0.0;
    for (int j = 0; j < H; ++j) {
        double inner = 0.0;
        for (int64_t n = n_lo; n < n_hi; ++n) {
            double st = 0.0;
            for (int d = 0; d < D; ++d) {
                double qd = bf(q[(int64_t)j * D + d]);
                double a = qd * bf(kmm_seq[n * 2 * D + d]);      /* q * k_max */
                double b = qd * bf(kmm_seq[n * 2 * D + D + d]);  /* q * k_min */
                st += a > b ? a : b;
            }
            if (st > 0.0) inner += st;
        }
        I += bf(w[j]) * inner;
    }
    return I;
}

/* Pages eligible for stage 1: those intersecting dyn = [lo, hi). */
static void eligible_pages(int64_t lo, int64_t hi, int P, int64_t *p0, int64_t *p1)
{
    if (hi <= lo) { *p0 = 0; *p1 = 0; return; }
    *p0 = lo / P;
    *p1 = (hi - 1) / P + 1;
}

/* --------------------------------- a1..a6: one query of the LSA indexer
 * Flat (M == 0): S_sparse = arg topK over dyn of Eq. 1 (Sec. 3.1).
 * Hierarchical (M > 0): rank eligible pages by Eq. 9, keep the top M (ties to
 * the lower page id), then Eq. 10 on the tokens of the recalled pages that
 * lie in dyn, then Eq. 11's arg topK (Sec. 3.3).
 * k_seq / kmean_seq point at this sequence's caches; L = its length.
 * Returns the number of valid indices written to out[0..K).
 */
int64_t orc_index_query_pool(const uint16_t *q, const uint16_t *w, const uint16_t *k_seq,
                             const uint16_t *kpool_seq, int pooling, int H, int D, int64_t L,
                             int64_t t, int K, int Ks, int Kw, int P, int B, int M,
                             int32_t *out);

int64_t orc_index_query(const uint16_t *q, const uint16_t *w, const uint16_t *k_seq,
                        const uint16_t *kmean_seq, int H, int D, int64_t L, int64_t t,
                        int K, int Ks, int Kw, int P, int B, int M, int32_t *out)
{
    return orc_index_query_pool(q, w, k_seq, kmean_seq, 0, H, D, L, t, K, Ks, Kw, P, B, M,
                                out);
}

/* The same indexer with the stage-1 pooling named: pooling 0 = mean (Eq. 9 on
 * kpool_seq = the sub-block means, rows of D), 1 = MinMax (Sec. 5.3.5 on
 * kpool_seq = the (k_max, k_min) rows of 2D).  Stage 2 is the same for both. */
int64_t orc_index_query_pool(const uint16_t *q, const uint16_t *w, const uint16_t *k_seq,
                             const uint16_t *kpool_seq, int pooling, int H, int D, int64_t L,
                             int64_t t, int K, int Ks, int Kw, int P, int B, int M,
                             int32_t *out)
{
    int64_t r[6];
    (void)L;
    orc_regions(t, Ks, Kw, r);
    int64_t lo = r[4], hi = r[5];
    int64_t n_dom = 0;
    int64_t *dom = NULL;
    if (M > 0) {
        int64_t p0, p1;
        eligible_pages(lo, hi, P, &p0, &p1);
        int64_t np = p1 - p0;
        int64_t *pid = (int64_t *)malloc(sizeof(int64_t) * (size_t)(np > 0 ? np : 1));
        double *ps = (double *)malloc(sizeof(double) * (size_t)(np > 0 ? np : 1));
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)M);
        for (int64_t i = 0; i < np; ++i) {
            pid[i] = p0 + i;
            ps[i] = pooling == 1
                        ? orc_page_score_minmax(q, w, kpool_seq, H, D, L, P, B, p0 + i)
                        : orc_page_score(q, w, kpool_seq, H, D, L, P, B, p0 + i);
        }
        int64_t mp = orc_topk(ps, pid, np, M, sel);
        dom = (int64_t *)malloc(sizeof(int64_t) * (size_t)(mp * P > 0 ? mp * P : 1));
        for (int64_t i = 0; i < mp; ++i) {
            int64_t a = (int64_t)sel[i] * P, b = a + P;
            if (a < lo) a = lo;
            if (b > hi) b = hi;
            for (int64_t s = a; s < b; ++s) dom[n_dom++] = s;
        }
        free(pid);
        free(ps);
        free(sel);
    } else {
        n_dom = hi - lo;
        dom = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_dom > 0 ? n_dom : 1));
        for (int64_t i = 0; i < n_dom; ++i) dom[i] = lo + i;
    }
    double *sc = (double *)malloc(sizeof(double) * (size_t)(n_dom > 0 ? n_dom : 1));
    orc_scores(q, w, k_seq, H, D, dom, n_dom, sc);
    int64_t m = orc_topk(sc, dom, n_dom, K, out);
    free(sc);
    free(dom);
    return m;
}

/* Batched indexer: q [B,T,H,D], w [B,T,H], k [B,Lmax,D], kmean [B,NBmax,D]
 * (NBmax = ceil(Lmax/Bsub)), kv_len [B], q_pos [B,T] -> out [B,T,K].
 * Independent (b, t) rows run in parallel (OpenMP). */
void orc_index_pool(const uint16_t *q, const uint16_t *w, const uint16_t *k,
                    const uint16_t *kpool, int pooling, const int32_t *kv_len,
                    const int32_t *q_pos, int Bn, int T, int H, int D, int64_t Lmax, int K,
                    int Ks, int Kw, int P, int Bsub, int M, int32_t *out)
{
    int64_t nbmax = (Bsub > 0) ? (Lmax + Bsub - 1) / Bsub : 0;
    int64_t width = pooling == 1 ? 2 * (int64_t)D : D;  /* elements per pooled row */
    int64_t rows = (int64_t)Bn * T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t row = 0; row < rows; ++row) {
        int64_t b = row / T;
        orc_index_query_pool(q + row * H * D, w + row * H, k + b * Lmax * D,
                             kpool ? kpool + b * nbmax * width : NULL, pooling, H, D,
                             kv_len[b], q_pos[row], K, Ks, Kw, P, Bsub, M, out + row * K);
    }
}

void orc_index(const uint16_t *q, const uint16_t *w, const uint16_t *k,
               const uint16_t *kmean, const int32_t *kv_len, const int32_t *q_pos,
               int Bn, int T, int H, int D, int64_t Lmax, int K, int Ks, int Kw,
               int P, int Bsub, int M, int32_t *out)
{
    orc_index_pool(q, w, k, kmean, 0, kv_len, q_pos, Bn, T, H, D, Lmax, K, Ks, Kw, P, Bsub, M,
                   out);
}

/* ----------------------- selection from externally computed score tensors
 * Runs the selection steps (a3, and a5's page top-M) of one query on scores
 * supplied by the caller instead of recomputing them: tok_scores[pos] for
 * every token position of the domain, page_scores[p] for every eligible page
 * (ignored when M == 0).  Scores are fp32 as exported by a device; they are
 * widened exactly to double before ranking.
 */
int64_t orc_select_query(const float *tok_scores, const float *page_scores,
                         int64_t t, int K, int Ks, int Kw, int P, int M, int32_t *out)
{
    int64_t r[6];
    orc_regions(t, Ks, Kw, r);
    int64_t lo = r[4], hi = r[5];
    int64_t n_dom = 0;
    int64_t *dom;
    if (M > 0) {
        int64_t p0, p1;
        eligible_pages(lo, hi, P, &p0, &p1);
        int64_t np = p1 - p0;
        int64_t *pid = (int64_t *)malloc(sizeof(int64_t) * (size_t)(np > 0 ? np : 1));
        double *ps = (double *)malloc(sizeof(double) * (size_t)(np > 0 ? np : 1));
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)M);
        for (int64_t i = 0; i < np; ++i) { pid[i] = p0 + i; ps[i] = (double)page_scores[p0 + i]; }
        int64_t mp = orc_topk(ps, pid, np, M, sel);
        dom = (int64_t *)malloc(sizeof(int64_t) * (size_t)(mp * P > 0 ? mp * P : 1));
        for (int64_t i = 0; i < mp; ++i) {
            int64_t a = (int64_t)sel[i] * P, b = a + P;
            if (a < lo) a = lo;
            if (b > hi) b = hi;
            for (int64_t s = a; s < b; ++s) dom[n_dom++] = s;
        }
        free(pid);
        free(ps);
        free(sel);
    } else {
        n_dom = hi - lo;
        dom = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_dom > 0 ? n_dom : 1));
        for (int64_t i = 0; i < n_dom; ++i) dom[i] = lo + i;
    }
    double *sc = (double *)malloc(sizeof(double) * (size_t)(n_dom > 0 ? n_dom : 1));
    for (int64_t i = 0; i < n_dom; ++i) sc[i] = (double)tok_scores[dom[i]];
    int64_t m = orc_topk(sc, dom, n_dom, K, out);
    free(sc);
    free(dom);
    return m;
}

/* ------------------------------------------------------- a7: attention
 * Hybrid sparse attention of one query (Sec. 4.1.1, with Fig. 1: sink and
 * SWA tokens take part in the same softmax as the dynamic tokens).
 * z_s = scale * q_h . c_s over S_t = sink U swa U {idx >= 0};
 * lse_h = log sum_s exp z_s;  out_h = sum_s exp(z_s - lse_h) * c_s[0:Dv].
 * q: [H*Dqk], c_seq: [Lmax*Dqk] latent rows, idx: [K] (-1 = empty slot).
 * Positions are visited as a set: sink, then swa, then idx in given order;
 * a duplicate position (which valid inputs never contain) is counted once.
 */
static int64_t gather_set(int64_t t, int Ks, int Kw, const int32_t *idx, int K,
                          int64_t *S)
{
    int64_t r[6], n = 0;
    orc_regions(t, Ks, Kw, r);
    for (int64_t s = r[0]; s < r[1]; ++s) S[n++] = s;
    for (int64_t s = r[2]; s < r[3]; ++s) S[n++] = s;
    for (int i = 0; i < K; ++i) {
        if (idx[i] < 0) continue;
        int dup = 0;
        for (int64_t j = 0; j < n; ++j) if (S[j] == idx[i]) { dup = 1; break; }
        if (!dup) S[n++] = idx[i];
    }
    return n;
}

/* Dense softmax attention of one head over an explicit position list. */
static void attend_list(const uint16_t *qh, const uint16_t *c_seq, const int64_t *S,
                        int64_t n, int Dqk, int Dv, double scale, double *out, double *lse)
{
    if (n == 0) {
        for (int d = 0; d < Dv; ++d) out[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double *z = (double *)malloc(sizeof(double) * (size_t)n);
    double zmax = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        double dot = 0.0;
        const uint16_t *c = c_seq + S[i] * Dqk;
        for (int d = 0; d < Dqk; ++d) dot += bf(qh[d]) * bf(c[d]);
        z[i] = scale * dot;
        if (z[i] > zmax) zmax = z[i];
    }
    double sum = 0.0;
    for (int64_t i = 0; i < n; ++i) sum += exp(z[i] - zmax);
    double L = zmax + log(sum);
    for (int d = 0; d < Dv; ++d) out[d] = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double p = exp(z[i] - L);
        const uint16_t *c = c_seq + S[i] * Dqk;
        for (int d = 0; d < Dv; ++d) out[d] += p * bf(c[d]);
    }
    *lse = L;
    free(z);
}

void orc_attend_query(const uint16_t *q, const uint16_t *c_seq, const int32_t *idx, int K,
                      int64_t t, int Ks, int Kw, int H, int Dqk, int Dv, double scale,
                      double *out, double *lse)
{
    int64_t *S = (int64_t *)malloc(sizeof(int64_t) * (size_t)(Ks + Kw + K + 1));
    int64_t n = gather_set(t, Ks, Kw, idx, K, S);
    for (int h = 0; h < H; ++h)
        attend_list(q + (int64_t)h * Dqk, c_seq, S, n, Dqk, Dv, scale,
                    out + (int64_t)h * Dv, lse + h);
    free(S);
}

/* The same result computed as the pages' two branches (Sec. 4.1.1): a
 * contiguous branch over sink U swa and a sparse branch over the indices,
 * each normalised on its own, then merged by log-sum-exp rescaling:
 *   lse = log(e^lse_a + e^lse_b),  out = e^(lse_a-lse) out_a + e^(lse_b-lse) out_b.
 * Used to check that the merge equals one softmax over the disjoint union. */
void orc_attend_query_branches(const uint16_t *q, const uint16_t *c_seq, const int32_t *idx,
                               int K, int64_t t, int Ks, int Kw, int H, int Dqk, int Dv,
                               double scale, double *out, double *lse)
{
    int64_t r[6];
    orc_regions(t, Ks, Kw, r);
    int64_t *Sa = (int64_t *)malloc(sizeof(int64_t) * (size_t)(Ks + Kw + 1));
    int64_t *Sb = (int64_t *)malloc(sizeof(int64_t) * (size_t)(K + 1));
    int64_t na = 0, nb = 0;
    for (int64_t s = r[0]; s < r[1]; ++s) Sa[na++] = s;
    for (int64_t s = r[2]; s < r[3]; ++s) Sa[na++] = s;
    for (int i = 0; i < K; ++i) if (idx[i] >= 0) Sb[nb++] = idx[i];
    double *oa = (double *)malloc(sizeof(double) * (size_t)Dv);
    double *ob = (double *)malloc(sizeof(double) * (size_t)Dv);
    for (int h = 0; h < H; ++h) {
        double la, lb;
        attend_list(q + (int64_t)h * Dqk, c_seq, Sa, na, Dqk, Dv, scale, oa, &la);
        attend_list(q + (int64_t)h * Dqk, c_seq, Sb, nb, Dqk, Dv, scale, ob, &lb);
        double m = la > lb ? la : lb;
        double L = (m == -INFINITY) ? -INFINITY : m + log(exp(la - m) + exp(lb - m));
        double *o = out + (int64_t)h * Dv;
        for (int d = 0; d < Dv; ++d) {
            double ca = (la == -INFINITY) ? 0.0 : exp(la - L);
            double cb = (lb == -INFINITY) ? 0.0 : exp(lb - L);
            o[d] = ca * oa[d] + cb * ob[d];
        }
        lse[h] = L;
    }
    free(Sa);
    free(Sb);
    free(oa);
    free(ob);
}

/* Batched attention: q [B,T,H,Dqk], c [B,Lmax,Dqk], idx [B,T,K], q_pos [B,T]
 * -> out [B,T,H,Dv] doubles, lse [B,T,H].  Rows in parallel (OpenMP).
 * A Cross-Layer-Indexing reuse layer (Sec. 3.2) is this same call with the
 * owner layer's idx array and its own q / c. */
void orc_attend(const uint16_t *q, const uint16_t *c, const int32_t *idx, const int32_t *q_pos,
                int Bn, int T, int H, int Dqk, int Dv, int64_t Lmax, int K, int Ks, int Kw,
                double scale, double *out, double *lse)
{
    int64_t rows = (int64_t)Bn * T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t row = 0; row < rows; ++row) {
        int64_t b = row / T;
        orc_attend_query(q + row * H * Dqk, c + b * Lmax * Dqk, idx + row * K, K,
                         q_pos[row], Ks, Kw, H, Dqk, Dv, scale,
                         out + row * H * Dv, lse + row * H);
    }
}

/* ---------------------------------------------------------------- FP8 indexer
 * The pages say only that the indexer can run in FP8 (Sec. 2.2, "Why Lightning") and
 * that DSA lowers its cost by FP8 quantization (Sec. 1).  Reading taken
 * (listed in the design notes): OCP E4M3 codes -- 1 sign bit, 4 exponent bits with bias
 * 7, 3 mantissa bits, no infinities, largest finite value 448, subnormals (m/8) * 2^-6 --
 * with one fp32 scale per row.  A key row is one token's d_I values, a query row is one
 * (token, head) vector.  For a row x: amax = max|x_i|, scale = amax / 448 and
 * code_i = nearest E4M3 value to x_i / scale (ties to the even code, saturated to
 * +-448), both quotients taken in IEEE fp32; an all-zero row has scale 0 and zero codes.
 * The score of key s for query t is Eq. 1 on the decoded rows:
 *   I[t,s] = sum_j w[t,j] * max(0, qs[t,j] * ks[s] * (q8[t,j] . k8[s])).
 */

/* value of an E4M3 code (0x7F / 0xFF are NaN and never produced) */
double orc_e4m3_value(uint8_t c)
{
    const int e = (c >> 3) & 0xF, m = c & 7;
    double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/* nearest E4M3 code to y: every non-negative finite code is tried; ties go to the code
 * with an even mantissa; |y| >= 448 saturates to 448 */
uint8_t orc_e4m3_encode(float y)
{
    const uint8_t sign = (y < 0.f || (y == 0.f && signbit(y))) ? 0x80 : 0;
    const double a = fabs((double)y);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    uint8_t best = 0;
    double best_d = a;  /* distance to code 0 */
    for (int c = 1; c <= 0x7E; ++c) {
        const double d = fabs(orc_e4m3_value((uint8_t)c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = (uint8_t)c;
            best_d = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* rows x[rows][D] (bf16 bits) -> codes[rows][D], scales[rows] */
void orc_quantize_e4m3(const uint16_t *x, int64_t rows, int D, uint8_t *codes, float *scales)
{
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *xr = x + r * D;
        float amax = 0.f;
        for (int i = 0; i < D; ++i) {
            const float v = fabsf((float)bf(xr[i]));
            if (v > amax) amax = v;
        }
        const float scale = amax / 448.0f;
        scales[r] = scale;
        for (int i = 0; i < D; ++i)
            codes[r * D + i] = (scale > 0.f) ? orc_e4m3_encode((float)bf(xr[i]) / scale) : 0;
    }
}

/* Eq. 1 on decoded FP8 rows: q8[H][D] codes with qs[H], w[H] (bf16 bits), key k8[D] with ks */
double orc_score_one_fp8(const uint8_t *q8, const float *qs, const uint16_t *w,
                         const uint8_t *k8, float ks, int H, int D)
{
    double s = 0.0;
    for (int j = 0; j < H; ++j) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += orc_e4m3_value(q8[j * D + d]) * orc_e4m3_value(k8[d]);
        const double x = (double)qs[j] * (double)ks * dot;
        s += bf(w[j]) * (x > 0.0 ? x : 0.0);
    }
    return s;
}

void orc_scores_fp8(const uint8_t *q8, const float *qs, const uint16_t *w, const uint8_t *k8_seq,
                    const float *ks_seq, int H, int D, const int64_t *pos, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_score_one_fp8(q8, qs, w, k8_seq + pos[i] * D, ks_seq[pos[i]], H, D);
}

/* ---------------------------------------------------------------- a7 backward (HFA bwd)
 * Gradient of the attention of Sec. 2.2 / 4.1.1 with respect to the query and the latent
 * rows (the pages' training path, Sec. 4.1.1 "backward pass", Table 2), by the textbook
 * rules of softmax attention over S_t (the same set as the forward):
 *   z_s = scale * q . c_s,  p_s = exp(z_s - lse),  o = sum_s p_s v_s  (v_s = c_s[0:Dv])
 *   dp_s = dout . v_s,  D = sum_s p_s dp_s,  dz_s = p_s (dp_s - D)
 *   dq   = scale * sum_s dz_s c_s                   (all Dqk dims)
 *   dc_s += scale * dz_s q  (all Dqk dims)  +  p_s dout  (first Dv dims)
 * Every quantity is fp64, recomputed from q and the rows (lse included).  A row selected by
 * several queries accumulates all their contributions. */
static void attend_bwd_list(const uint16_t *qh, const uint16_t *c_seq, const int64_t *S,
                            int64_t n, int Dqk, int Dv, double scale, const double *dout,
                            double *dq, double *dc_seq)
{
    for (int d = 0; d < Dqk; ++d) dq[d] = 0.0;
    if (n == 0) return;
    double *z = (double *)malloc(sizeof(double) * (size_t)n);
    double *dp = (double *)malloc(sizeof(double) * (size_t)n);
    double zmax = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        double dot = 0.0;
        const uint16_t *c = c_seq + S[i] * Dqk;
        for (int d = 0; d < Dqk; ++d) dot += bf(qh[d]) * bf(c[d]);
        z[i] = scale * dot;
        if (z[i] > zmax) zmax = z[i];
        double g = 0.0;
        for (int d = 0; d < Dv; ++d) g += dout[d] * bf(c[d]);
        dp[i] = g;
    }
    double sum = 0.0;
    for (int64_t i = 0; i < n; ++i) sum += exp(z[i] - zmax);
    const double L = zmax + log(sum);
    double D = 0.0;
    for (int64_t i = 0; i < n; ++i) D += exp(z[i] - L) * dp[i];
    for (int64_t i = 0; i < n; ++i) {
        const double p = exp(z[i] - L);
        const double dz = p * (dp[i] - D);
        const uint16_t *c = c_seq + S[i] * Dqk;
        double *g = dc_seq + S[i] * Dqk;
        for (int d = 0; d < Dqk; ++d) {
            dq[d] += scale * dz * bf(c[d]);
            g[d] += scale * dz * bf(qh[d]);
        }
        for (int d = 0; d < Dv; ++d) g[d] += p * dout[d];
    }
    free(z);
    free(dp);
}

/* One query row: q [H][Dqk], dout [H][Dv] (fp64) -> dq [H][Dqk]; dc_seq [L][Dqk] accumulated. */
void orc_attend_bwd_query(const uint16_t *q, const uint16_t *c_seq, const int32_t *idx, int K,
                          int64_t t, int Ks, int Kw, int H, int Dqk, int Dv, double scale,
                          const double *dout, double *dq, double *dc_seq)
{
    int64_t *S = (int64_t *)malloc(sizeof(int64_t) * (size_t)(Ks + Kw + K + 1));
    int64_t n = gather_set(t, Ks, Kw, idx, K, S);
    for (int h = 0; h < H; ++h)
        attend_bwd_list(q + (int64_t)h * Dqk, c_seq, S, n, Dqk, Dv, scale,
                        dout + (int64_t)h * Dv, dq + (int64_t)h * Dqk, dc_seq);
    free(S);
}

/* Batched: q [B][T][H][Dqk], c [B][Lmax][Dqk], idx [B][T][K], q_pos [B][T], dout [B][T][H][Dv]
 * -> dq [B][T][H][Dqk], dc [B][Lmax][Dqk] (zeroed here, then accumulated).  Sequences run in
 * parallel; the rows of one sequence run in order, so the sums are deterministic. */
void orc_attend_bwd(const uint16_t *q, const uint16_t *c, const int32_t *idx, const int32_t *q_pos,
                    int B, int T, int H, int Dqk, int Dv, int64_t Lmax, int K, int Ks, int Kw,
                    double scale, const double *dout, double *dq, double *dc)
{
    memset(dc, 0, sizeof(double) * (size_t)B * (size_t)Lmax * (size_t)Dqk);
    #pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < T; ++i) {
            const int64_t row = (int64_t)b * T + i;
            orc_attend_bwd_query(q + row * H * Dqk, c + (int64_t)b * Lmax * Dqk, idx + row * K, K,
                                 q_pos[row], Ks, Kw, H, Dqk, Dv, scale, dout + row * H * Dv,
                                 dq + row * H * Dqk, dc + (int64_t)b * Lmax * Dqk);
        }
}
