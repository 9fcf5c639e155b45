// lsa_api.cu -- the extern "C" boundary of liblsa.so (declared in include/lsa.h).
//
// Host side only: argument validation, workspace layout, and the launch sequence of each
// entry point.  Every step of the computation runs in the kernels of this library.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>

#include "lsa_internal.cuh"
#include "score_tc.cuh"

namespace lsa {
namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

struct IndexLayout {
    size_t err, hist, counts, sure, cand, scores, pscores, pages, pcount, s2, total;
    int64_t rows, n_pages, sel_cap, cand_slots;
};

bool index_args_ok(int B, int T, int H_I, int D_I, int64_t L_max, int K, int page, int sub,
                   int M) {
    if (B < 1 || T < 1 || H_I < 8 || H_I > 128 || H_I % 8) return false;
    if (D_I != 64 && D_I != 128) return false;
    if (L_max < 1 || L_max > 0x7FFFFFFFll) return false;
    if (K < 1 || K > kMaxSelect) return false;
    if (M < 0 || M > kMaxSelect) return false;
    if (M > 0) {
        if (page != 32 && page != 64 && page != 128 && page != 256) return false;
        if (sub < 1 || page % sub) return false;
    }
    return true;
}

IndexLayout index_layout(int B, int T, int64_t L_max, int K, int page, int M) {
    IndexLayout L;
    L.rows = (int64_t)B * T;
    L.n_pages = M > 0 ? (L_max + page - 1) / page : 0;
    L.sel_cap = K > M ? K : M;
    L.cand_slots = M > 0 ? (L.n_pages > (int64_t)M * page ? L.n_pages : (int64_t)M * page) : L_max;
    size_t off = 0;
    L.err = off;
    off += kAlign;
    L.hist = off;
    off = align_up(off + (size_t)L.rows * kHistBins * 4);
    L.counts = off;
    off = align_up(off + (size_t)L.rows * kCountStride * 4);
    L.sure = off;
    off = align_up(off + (size_t)L.rows * L.sel_cap * 4);
    L.cand = off;
    off = align_up(off + (size_t)L.rows * L.cand_slots * 4);
    L.scores = off;
    off = align_up(off + (M == 0 ? (size_t)L.rows * L_max * 4 : 0));
    L.pscores = off;
    off = align_up(off + (size_t)L.rows * L.n_pages * 4);
    L.pages = off;
    off = align_up(off + (size_t)L.rows * M * 4);
    L.pcount = off;
    off = align_up(off + (size_t)L.rows * 4);
    L.s2 = off;
    off = align_up(off + (size_t)L.rows * M * page * 4);
    L.total = off;
    return L;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

struct AttendPlan {
    int n_split, tiles_per_split;
    size_t err, part_o, part_lse, total;
};

// Key-split plan of lsa_attend: enough splits that the grid covers the SMs once.
AttendPlan attend_plan(int B, int T, int H, int K, int sink, int swa, bool tc) {
    AttendPlan p;
    const int64_t rows = (int64_t)B * T;
    const int64_t tile = tc ? attend_tc_tile() : 32;
    const int hg = attend_heads_per_cta(H);
    const int64_t groups = tc ? 2 : (H + hg - 1) / hg;
    const int64_t tiles = ((int64_t)sink + swa + K + tile - 1) / tile;
    const int64_t ctas = rows * groups;
    const int64_t sms = num_sms();
    int64_t ns = ctas >= sms ? 1 : sms / ctas;
    if (ns > tiles) ns = tiles;
    if (ns < 1) ns = 1;
    int64_t tps = (tiles + ns - 1) / ns;
    if (tps < 1) tps = 1;
    ns = (tiles + tps - 1) / tps;
    if (ns < 1) ns = 1;
    p.n_split = (int)ns;
    p.tiles_per_split = (int)tps;
    size_t off = 0;
    p.err = off;
    off += kAlign;
    p.part_o = off;
    off = align_up(off + (ns > 1 ? (size_t)rows * H * ns * 512 * 4 : 0));
    p.part_lse = off;
    off = align_up(off + (ns > 1 ? (size_t)rows * H * ns * 4 : 0));
    p.total = off;
    return p;
}

// LSA_NO_TCGEN05=1 selects the CUDA-core scorer and the mma.sync attention kernels (forward and
// backward) even where the tcgen05 kernels apply (both families are tested against the oracle).
bool tc_allowed() {
    const char *v = getenv("LSA_NO_TCGEN05");
    return !(v && v[0] == '1');
}

bool attend_uses_tc(int H) { return H == 128 && tc_allowed(); }

// LSA_SCORE_ONE_QUERY=1 scores prefill rows with the one-query tensor-core kernel instead of the
// multi-query one (both are tested against the oracle).
bool mq_allowed() {
    const char *v = getenv("LSA_SCORE_ONE_QUERY");
    return !(v && v[0] == '1');
}

TcScoreArgs tc_args(const ScoreArgs &sa, int64_t nb_max, uint32_t *hist) {
    TcScoreArgs t;
    memset(&t, 0, sizeof t);
    t.q = sa.q;
    t.w = sa.w;
    t.q_pos = sa.q_pos;
    t.kv_len = sa.kv_len;
    t.T = sa.T;
    t.H = sa.H;
    t.L_max = sa.L_max;
    t.nb_max = nb_max;
    t.Ks = sa.Ks;
    t.Kw = sa.Kw;
    t.P = sa.P;
    t.Bsub = sa.Bsub;
    t.mode = sa.mode;
    t.minmax = sa.minmax;
    t.page_list = sa.page_list;
    t.page_count = sa.page_count;
    t.page_stride = sa.page_stride;
    t.out = sa.out;
    t.out_stride = sa.out_stride;
    t.hist = hist;
    t.err = sa.err;
    return t;
}

// Scores one scoring pass and runs the matching selection: the tensor-core kernel (which also
// builds the selection histogram) where it applies, else the CUDA-core kernel.
// cleared: the row histograms and counters are already zero (the entry point clears them with
// its error word in one memset before the first pass).
cudaError_t score_and_select(const ScoreArgs &sa, const SelectArgs &se, int64_t rows,
                             int64_t max_units, int64_t max_slots, int64_t key_rows,
                             int64_t nb_max, int64_t max_tiles, cudaStream_t s,
                             bool cleared = false) {
    cudaError_t e;
    // rows the one-launch select takes need no first-digit histogram from the scorer
    const bool small = select_is_small(rows, max_slots);
    if (tc_allowed() && mq_allowed() &&
        mq_score_supported(sa.H, sa.D, sa.T, sa.mode, sa.P, sa.Bsub, sa.minmax) &&
        rows / sa.T * ((sa.T + 1) / 2) <= 65535 &&
        tc_score_supported(sa.H, sa.D, sa.mode, sa.P, sa.Bsub, key_rows)) {
        // several queries of a sequence per CTA (prefill)
        if (!small && !cleared && (e = select_clear(se, rows, s)) != cudaSuccess) return e;
        TcScoreArgs ta = tc_args(sa, nb_max, small ? nullptr : se.hist);
        ta.counts = se.counts;
        ta.sel_K = se.K;
        if ((e = launch_score_mq(ta, sa.keys, key_rows, (int)(rows / sa.T), max_tiles, s)) !=
            cudaSuccess)
            return e;
        SelectArgs se2 = se;
        se2.thr_ready = 1;
        return launch_select(se2, rows, max_slots, s, true);
    }
    if (tc_allowed() && rows <= 65535 &&
        tc_score_supported(sa.H, sa.D, sa.mode, sa.P, sa.Bsub, key_rows)) {
        if (!small && !cleared && (e = select_clear(se, rows, s)) != cudaSuccess) return e;
        TcScoreArgs ta = tc_args(sa, nb_max, small ? nullptr : se.hist);
        ta.counts = se.counts;
        ta.sel_K = se.K;
        if ((e = launch_score_tc(ta, sa.keys, key_rows, sa.D, rows, max_tiles, s)) != cudaSuccess)
            return e;
        SelectArgs se2 = se;
        se2.thr_ready = 1;
        return launch_select(se2, rows, max_slots, s, true);
    }
    if ((e = launch_score(sa, rows, max_units, s)) != cudaSuccess) return e;
    return launch_select(se, rows, max_slots, s, false);
}

// True when p (may be null) is not a multiple of `align` bytes.  The kernels read bf16 rows with
// 16-byte vector loads, cp.async and TMA, so such a pointer would fault on the device instead of
// failing here.
inline bool misaligned(const void *p, uintptr_t align) {
    return (reinterpret_cast<uintptr_t>(p) % align) != 0;
}

lsa_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return LSA_OK;
    cudaGetLastError();
    return LSA_ERR_CUDA;
}

// HI stage-2 scores are kept per recalled-page slot; the debug export scatters them to
// absolute positions.
__global__ void export_stage2_kernel(const float *s2, const int32_t *pages, const int32_t *pcount,
                                     int M, int P, int64_t L_max, float *dbg) {
    const int64_t r = blockIdx.y;
    const int64_t n = (int64_t)pcount[r] * P;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < n;
         u += (int64_t)gridDim.x * blockDim.x) {
        const float v = s2[r * (int64_t)M * P + u];
        if (__float_as_uint(v) == kExcludedBits) continue;
        const int64_t pos = (int64_t)pages[r * M + u / P] * P + u % P;
        dbg[r * L_max + pos] = v;
    }
}

}  // namespace

std::atomic<uint64_t> g_launches{0};

cudaError_t launched() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace lsa

using namespace lsa;

// The indexer behind lsa_index (pooling 0: k_pool = sub-block means, D_I wide) and
// lsa_index_minmax (pooling 1: k_pool = MinMax rows, 2 D_I wide; tensor-core scorer only).
static lsa_status index_impl(const void *q_I, const void *w_I, const void *k_I,
                             const void *k_pool, int pooling, const int32_t *kv_len,
                             const int32_t *q_pos, int B, int T, int H_I, int D_I, int64_t L_max,
                             int K_sparse, int sink, int swa, int page, int sub_block, int M,
                             int32_t *indices, float *scores_dbg, float *page_scores_dbg,
                             void *ws, size_t ws_bytes, void *stream) {
    const void *k_mean = k_pool;
    if (!q_I || !w_I || !k_I || !kv_len || !q_pos || !indices || !ws) return LSA_ERR_INVALID_ARG;
    if (sink < 0 || swa < 0 || B < 1 || T < 1 || L_max < 1 || K_sparse < 1 || M < 0)
        return LSA_ERR_INVALID_ARG;
    if (M > 0 && (!k_mean || page < 1 || sub_block < 1 || page % sub_block))
        return LSA_ERR_INVALID_ARG;
    if (!index_args_ok(B, T, H_I, D_I, L_max, K_sparse, page, sub_block, M))
        return LSA_ERR_UNSUPPORTED;
    if (misaligned(ws, 16) || misaligned(q_I, 16) || misaligned(k_I, 16) ||
        (M > 0 && misaligned(k_mean, 16)) || misaligned(w_I, 2) || misaligned(kv_len, 4) ||
        misaligned(q_pos, 4) || misaligned(indices, 4) || misaligned(scores_dbg, 4) ||
        misaligned(page_scores_dbg, 4))
        return LSA_ERR_INVALID_ARG;
    const IndexLayout L = index_layout(B, T, L_max, K_sparse, page, M);
    if (ws_bytes < L.total) return LSA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    int32_t *err = reinterpret_cast<int32_t *>(w8 + L.err);
    // the error word, the row histograms and the row counters are contiguous: one memset
    cudaError_t e = cudaMemsetAsync(err, 0, L.counts + (size_t)L.rows * kCountStride * 4, s);
    if (e != cudaSuccess) return cuda_status(e);

    ScoreArgs sa;
    memset(&sa, 0, sizeof sa);
    sa.q = static_cast<const __nv_bfloat16 *>(q_I);
    sa.w = static_cast<const __nv_bfloat16 *>(w_I);
    sa.q_pos = q_pos;
    sa.kv_len = kv_len;
    sa.T = T;
    sa.H = H_I;
    sa.D = D_I;
    sa.L_max = L_max;
    sa.Ks = sink;
    sa.Kw = swa;
    sa.P = page;
    sa.Bsub = sub_block;
    sa.err = err;

    SelectArgs se;
    memset(&se, 0, sizeof se);
    se.q_pos = q_pos;
    se.kv_len = kv_len;
    se.T = T;
    se.L_max = L_max;
    se.Ks = sink;
    se.Kw = swa;
    se.P = page;
    se.hist = reinterpret_cast<uint32_t *>(w8 + L.hist);
    se.counts = reinterpret_cast<int32_t *>(w8 + L.counts);
    se.sure = reinterpret_cast<int32_t *>(w8 + L.sure);
    se.sure_stride = (int)L.sel_cap;
    se.cand = reinterpret_cast<int32_t *>(w8 + L.cand);
    se.cand_stride = L.cand_slots;
    se.err = err;

    if (M == 0) {
        float *scores = scores_dbg ? scores_dbg : reinterpret_cast<float *>(w8 + L.scores);
        sa.keys = static_cast<const __nv_bfloat16 *>(k_I);
        sa.key_seq_stride = L_max * D_I;
        sa.mode = kScoreTokens;
        sa.out = scores;
        sa.out_stride = L_max;
        se.scores = scores;
        se.row_stride = L_max;
        se.mode = kSelTokens;
        se.K = K_sparse;
        se.out = indices;
        se.out_stride = K_sparse;
        e = score_and_select(sa, se, L.rows, L_max, L_max, (int64_t)B * L_max, 0,
                             (L_max + 127) / 128, s, true);
        return cuda_status(e);
    }

    // ---- Hierarchical Indexing: stage 1 (Eq. 9) -> top-M pages -> stage 2 (Eq. 10/11)
    float *pscores =
        page_scores_dbg ? page_scores_dbg : reinterpret_cast<float *>(w8 + L.pscores);
    int32_t *pages = reinterpret_cast<int32_t *>(w8 + L.pages);
    int32_t *pcount = reinterpret_cast<int32_t *>(w8 + L.pcount);
    float *s2 = reinterpret_cast<float *>(w8 + L.s2);
    const int64_t nbmax = (L_max + sub_block - 1) / sub_block;

    sa.keys = static_cast<const __nv_bfloat16 *>(k_mean);
    sa.key_seq_stride = nbmax * D_I * (pooling == 1 ? 2 : 1);
    sa.mode = kScorePages;
    sa.minmax = pooling == 1 ? 1 : 0;
    sa.out = pscores;
    sa.out_stride = L.n_pages;
    se.scores = pscores;
    se.row_stride = L.n_pages;
    se.mode = kSelPages;
    se.K = M;
    se.out = pages;
    se.out_stride = M;
    se.out_count = pcount;
    {
        const int64_t per = page / sub_block;
        e = score_and_select(sa, se, L.rows, L.n_pages, L.n_pages, (int64_t)B * nbmax, nbmax,
                             (L.n_pages * per + 127) / 128, s, true);
        if (e != cudaSuccess) return cuda_status(e);
    }

    sa.keys = static_cast<const __nv_bfloat16 *>(k_I);
    sa.key_seq_stride = L_max * D_I;
    sa.mode = kScoreStage2;
    sa.minmax = 0;
    sa.page_list = pages;
    sa.page_count = pcount;
    sa.page_stride = M;
    sa.out = s2;
    sa.out_stride = (int64_t)M * page;
    se.scores = s2;
    se.row_stride = (int64_t)M * page;
    se.mode = kSelStage2;
    se.page_list = pages;
    se.page_count = pcount;
    se.page_stride = M;
    se.K = K_sparse;
    se.out = indices;
    se.out_stride = K_sparse;
    se.out_count = nullptr;
    e = score_and_select(sa, se, L.rows, (int64_t)M * page, (int64_t)M * page,
                         (int64_t)B * L_max, 0, M, s);
    if (e != cudaSuccess) return cuda_status(e);

    if (scores_dbg) {
        for (int64_t r0 = 0; r0 < L.rows; r0 += 65535) {
            const int64_t nr = L.rows - r0 < 65535 ? L.rows - r0 : 65535;
            dim3 grid(256, (unsigned)nr);
            export_stage2_kernel<<<grid, 256, 0, s>>>(
                s2 + r0 * (int64_t)M * page, pages + r0 * M, pcount + r0, M, page, L_max,
                scores_dbg + r0 * L_max);
            if ((e = launched()) != cudaSuccess) return cuda_status(e);
        }
    }
    return LSA_OK;
}

extern "C" {

const char *lsa_status_string(lsa_status s) {
    switch (s) {
        case LSA_OK: return "LSA_OK";
        case LSA_ERR_INVALID_ARG: return "LSA_ERR_INVALID_ARG";
        case LSA_ERR_UNSUPPORTED: return "LSA_ERR_UNSUPPORTED";
        case LSA_ERR_WORKSPACE: return "LSA_ERR_WORKSPACE";
        case LSA_ERR_CUDA: return "LSA_ERR_CUDA";
        case LSA_ERR_DEVICE: return "LSA_ERR_DEVICE";
    }
    return "LSA_ERR_UNKNOWN";
}

int lsa_version(void) { return 100; }

uint64_t lsa_launch_count(void) { return lsa::g_launches.load(std::memory_order_relaxed); }

size_t lsa_index_workspace_bytes(int B, int T, int H_I, int D_I, int64_t L_max, int K_sparse,
                                 int page, int sub_block, int M) {
    if (!index_args_ok(B, T, H_I, D_I, L_max, K_sparse, page, sub_block, M)) return 0;
    return index_layout(B, T, L_max, K_sparse, page, M).total;
}

lsa_status lsa_index(const void *q_I, const void *w_I, const void *k_I, const void *k_mean,
                     const int32_t *kv_len, const int32_t *q_pos, int B, int T, int H_I, int D_I,
                     int64_t L_max, int K_sparse, int sink, int swa, int page, int sub_block,
                     int M, int32_t *indices, float *scores_dbg, float *page_scores_dbg,
                     void *ws, size_t ws_bytes, void *stream) {
    return index_impl(q_I, w_I, k_I, k_mean, 0, kv_len, q_pos, B, T, H_I, D_I, L_max, K_sparse,
                      sink, swa, page, sub_block, M, indices, scores_dbg, page_scores_dbg, ws,
                      ws_bytes, stream);
}

lsa_status lsa_index_minmax(const void *q_I, const void *w_I, const void *k_I,
                            const void *k_minmax, const int32_t *kv_len, const int32_t *q_pos,
                            int B, int T, int H_I, int D_I, int64_t L_max, int K_sparse, int sink,
                            int swa, int page, int sub_block, int M, int32_t *indices,
                            float *scores_dbg, float *page_scores_dbg, void *ws, size_t ws_bytes,
                            void *stream) {
    if (M < 1 || !k_minmax) return LSA_ERR_INVALID_ARG;
    if (!index_args_ok(B, T, H_I, D_I, L_max, K_sparse, page, sub_block, M))
        return LSA_ERR_UNSUPPORTED;
    // the MinMax page score exists only on the tensor cores (H_I in {64, 128})
    const int64_t nbmax = (L_max + sub_block - 1) / sub_block;
    if (!tc_allowed() || (int64_t)B * T > 65535 ||
        !tc_score_supported(H_I, D_I, kScorePages, page, sub_block, (int64_t)B * nbmax))
        return LSA_ERR_UNSUPPORTED;
    return index_impl(q_I, w_I, k_I, k_minmax, 1, kv_len, q_pos, B, T, H_I, D_I, L_max,
                      K_sparse, sink, swa, page, sub_block, M, indices, scores_dbg,
                      page_scores_dbg, ws, ws_bytes, stream);
}

lsa_status lsa_index_fp8(const uint8_t *q8, const float *q_scale, const void *w_I,
                         const uint8_t *k8, const float *k_scale, const int32_t *kv_len,
                         const int32_t *q_pos, int B, int T, int H_I, int D_I, int64_t L_max,
                         int K_sparse, int sink, int swa, int32_t *indices, float *scores_dbg,
                         void *ws, size_t ws_bytes, void *stream) {
    if (!q8 || !q_scale || !w_I || !k8 || !k_scale || !kv_len || !q_pos || !indices || !ws)
        return LSA_ERR_INVALID_ARG;
    if (sink < 0 || swa < 0 || B < 1 || T < 1 || L_max < 1 || K_sparse < 1)
        return LSA_ERR_INVALID_ARG;
    if (misaligned(ws, 16) || misaligned(q8, 16) || misaligned(k8, 16) || misaligned(w_I, 2) ||
        misaligned(q_scale, 4) || misaligned(k_scale, 4) || misaligned(kv_len, 4) ||
        misaligned(q_pos, 4) || misaligned(indices, 4) || misaligned(scores_dbg, 4))
        return LSA_ERR_INVALID_ARG;
    if (!index_args_ok(B, T, H_I, D_I, L_max, K_sparse, 128, 8, 0)) return LSA_ERR_UNSUPPORTED;
    // the FP8 scorer exists only on the tensor cores: d_I = 128 (one 128-byte code row per key)
    if (D_I != 128 || !(H_I == 64 || H_I == 128) || (int64_t)B * T > 65535 ||
        !tc_score_supported(H_I, D_I, kScoreTokens, 128, 8, (int64_t)B * L_max))
        return LSA_ERR_UNSUPPORTED;
    const IndexLayout L = index_layout(B, T, L_max, K_sparse, 128, 0);
    if (ws_bytes < L.total) return LSA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    int32_t *err = reinterpret_cast<int32_t *>(w8 + L.err);
    // the error word, the row histograms and the row counters are contiguous: one memset
    cudaError_t e = cudaMemsetAsync(err, 0, L.counts + (size_t)L.rows * kCountStride * 4, s);
    if (e != cudaSuccess) return cuda_status(e);
    float *scores = scores_dbg ? scores_dbg : reinterpret_cast<float *>(w8 + L.scores);

    SelectArgs se;
    memset(&se, 0, sizeof se);
    se.q_pos = q_pos;
    se.kv_len = kv_len;
    se.T = T;
    se.L_max = L_max;
    se.Ks = sink;
    se.Kw = swa;
    se.P = 128;
    se.hist = reinterpret_cast<uint32_t *>(w8 + L.hist);
    se.counts = reinterpret_cast<int32_t *>(w8 + L.counts);
    se.sure = reinterpret_cast<int32_t *>(w8 + L.sure);
    se.sure_stride = (int)L.sel_cap;
    se.cand = reinterpret_cast<int32_t *>(w8 + L.cand);
    se.cand_stride = L.cand_slots;
    se.err = err;
    se.scores = scores;
    se.row_stride = L_max;
    se.mode = kSelTokens;
    se.K = K_sparse;
    se.out = indices;
    se.out_stride = K_sparse;

    TcScoreArgs ta;
    memset(&ta, 0, sizeof ta);
    ta.q8 = q8;
    ta.qscale = q_scale;
    ta.kscale = k_scale;
    ta.w = static_cast<const __nv_bfloat16 *>(w_I);
    ta.q_pos = q_pos;
    ta.kv_len = kv_len;
    ta.T = T;
    ta.H = H_I;
    ta.L_max = L_max;
    ta.Ks = sink;
    ta.Kw = swa;
    ta.P = 128;
    ta.Bsub = 8;
    ta.mode = kScoreTokens;
    ta.out = scores;
    ta.out_stride = L_max;
    // rows the one-launch select takes need no first-digit histogram from the scorer
    ta.hist = select_is_small(L.rows, L_max) ? nullptr : se.hist;
    ta.counts = se.counts;
    ta.sel_K = K_sparse;
    ta.err = err;
    if ((e = launch_score_tc_fp8(ta, k8, (int64_t)B * L_max, D_I, L.rows, (L_max + 127) / 128,
                                 s)) != cudaSuccess)
        return cuda_status(e);
    se.thr_ready = 1;
    return cuda_status(launch_select(se, L.rows, L_max, s, true));
}

lsa_status lsa_attend_bwd(const void *q, const void *c_kv, const int32_t *indices,
                          const int32_t *kv_len, const int32_t *q_pos, int B, int T, int H,
                          int D_qk, int D_v, int64_t L_max, int K_sparse, int sink, int swa,
                          float scale, const void *out, const float *lse, const void *dout,
                          float *dq, float *dc_kv, int32_t *device_error, void *stream) {
    if (!q || !c_kv || !kv_len || !q_pos || !dout || !dq || !dc_kv) return LSA_ERR_INVALID_ARG;
    if ((out == nullptr) != (lse == nullptr)) return LSA_ERR_INVALID_ARG;
    if (K_sparse > 0 && !indices) return LSA_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1 || L_max < 1 || K_sparse < 0 || sink < 0 || swa < 0)
        return LSA_ERR_INVALID_ARG;
    if (!(scale > 0.f && scale <= 3.4e38f)) return LSA_ERR_INVALID_ARG;
    if (H % 32 || D_qk != 576 || D_v != 512 || K_sparse > kMaxSelect || L_max > 0x7FFFFFFFll ||
        (int64_t)B * T > 0x7FFFFFFF || H / 32 > 65535)
        return LSA_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(c_kv) % 16 ||
        reinterpret_cast<uintptr_t>(dout) % 16 || reinterpret_cast<uintptr_t>(dq) % 8 ||
        reinterpret_cast<uintptr_t>(dc_kv) % 16 || reinterpret_cast<uintptr_t>(out) % 16 ||
        reinterpret_cast<uintptr_t>(lse) % 4)
        return LSA_ERR_INVALID_ARG;
    BwdArgs a;
    memset(&a, 0, sizeof a);
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.c = static_cast<const __nv_bfloat16 *>(c_kv);
    a.idx = indices;
    a.kv_len = kv_len;
    a.q_pos = q_pos;
    a.dout = static_cast<const __nv_bfloat16 *>(dout);
    a.o = static_cast<const __nv_bfloat16 *>(out);
    a.lse = lse;
    a.dq = dq;
    a.dc = dc_kv;
    a.T = T;
    a.H = H;
    a.K = K_sparse;
    a.Ks = sink;
    a.Kw = swa;
    a.L_max = L_max;
    a.scale = scale;
    a.err = device_error;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tc_allowed() && attend_bwd_tc_supported(a))
        return cuda_status(launch_attend_bwd_tc(a, (int64_t)B * T, s));
    return cuda_status(launch_attend_bwd(a, (int64_t)B * T, s));
}

size_t lsa_attend_workspace_bytes(int B, int T, int H, int D_v, int K_sparse, int sink, int swa) {
    if (B < 1 || T < 1 || H < 8 || H > 128 || H % 8 || D_v != 512 || K_sparse < 0 ||
        K_sparse > kMaxSelect || sink < 0 || swa < 0)
        return 0;
    size_t n = attend_plan(B, T, H, K_sparse, sink, swa, false).total;
    if (H == 128) {
        const size_t m = attend_plan(B, T, H, K_sparse, sink, swa, true).total;
        if (m > n) n = m;
    }
    return n;
}

lsa_status lsa_attend(const void *q, const void *c_kv, const int32_t *indices,
                      const int32_t *kv_len, const int32_t *q_pos, int B, int T, int H, int D_qk,
                      int D_v, int64_t L_max, int K_sparse, int sink, int swa, float scale,
                      void *out, float *lse, void *ws, size_t ws_bytes, void *stream) {
    if (!q || !c_kv || !kv_len || !q_pos || !out || !lse || !ws) return LSA_ERR_INVALID_ARG;
    if (K_sparse > 0 && !indices) return LSA_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1 || L_max < 1 || K_sparse < 0 || sink < 0 || swa < 0)
        return LSA_ERR_INVALID_ARG;
    if (!(scale > 0.f && scale <= 3.4e38f)) return LSA_ERR_INVALID_ARG;  // positive, finite
    if (H > 128 || H % 8 || D_qk != 576 || D_v != 512 || K_sparse > kMaxSelect ||
        L_max > 0x7FFFFFFFll)
        return LSA_ERR_UNSUPPORTED;
    if (misaligned(ws, 16) || misaligned(q, 16) || misaligned(c_kv, 16) || misaligned(out, 16) ||
        misaligned(lse, 4) || misaligned(indices, 4) || misaligned(kv_len, 4) ||
        misaligned(q_pos, 4))
        return LSA_ERR_INVALID_ARG;
    const bool use_tc = attend_uses_tc(H);
    const AttendPlan p = attend_plan(B, T, H, K_sparse, sink, swa, use_tc);
    if (ws_bytes < p.total) return LSA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    int32_t *err = reinterpret_cast<int32_t *>(w8 + p.err);
    cudaError_t e = cudaMemsetAsync(err, 0, 4, s);
    if (e != cudaSuccess) return cuda_status(e);
    AttendArgs a;
    memset(&a, 0, sizeof a);
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.c = static_cast<const __nv_bfloat16 *>(c_kv);
    a.idx = indices;
    a.q_pos = q_pos;
    a.kv_len = kv_len;
    a.T = T;
    a.H = H;
    a.K = K_sparse;
    a.L_max = L_max;
    a.Ks = sink;
    a.Kw = swa;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.part_o = reinterpret_cast<float *>(w8 + p.part_o);
    a.part_lse = reinterpret_cast<float *>(w8 + p.part_lse);
    a.n_split = p.n_split;
    a.tiles_per_split = p.tiles_per_split;
    a.use_tc = use_tc ? 1 : 0;
    a.err = err;
    e = launch_attend(a, (int64_t)B * T, s);
    return cuda_status(e);
}

lsa_status lsa_kv_append(const void *k_I_new, void *k_I, void *k_mean, const void *c_new,
                         void *c_kv, const int32_t *kv_len_old, int B, int n_new, int D_I,
                         int D_qk, int64_t L_max, int sub_block, int32_t *device_error,
                         void *stream) {
    if (!kv_len_old || B < 1 || n_new < 0 || L_max < 1) return LSA_ERR_INVALID_ARG;
    if (!k_I_new && !c_new) return LSA_ERR_INVALID_ARG;
    if (k_I_new && !k_I) return LSA_ERR_INVALID_ARG;
    if (c_new && !c_kv) return LSA_ERR_INVALID_ARG;
    if (k_I_new && D_I != 64 && D_I != 128) return LSA_ERR_UNSUPPORTED;
    if (k_I_new && k_mean && (sub_block < 1 || sub_block > 4096)) return LSA_ERR_INVALID_ARG;
    if (c_new && (D_qk < 8 || D_qk % 8)) return LSA_ERR_UNSUPPORTED;
    if (B > 65535 || L_max > 0x7FFFFFFFll) return LSA_ERR_UNSUPPORTED;
    if (misaligned(k_I_new, 16) || misaligned(k_I, 16) || misaligned(k_mean, 16) ||
        misaligned(c_new, 16) || misaligned(c_kv, 16) || misaligned(kv_len_old, 4) ||
        misaligned(device_error, 4))
        return LSA_ERR_INVALID_ARG;
    if (n_new == 0) return LSA_OK;
    AppendArgs a;
    memset(&a, 0, sizeof a);
    a.k_new = static_cast<const __nv_bfloat16 *>(k_I_new);
    a.k = static_cast<__nv_bfloat16 *>(k_I);
    a.k_mean = static_cast<__nv_bfloat16 *>(k_mean);
    a.c_new = static_cast<const __nv_bfloat16 *>(c_new);
    a.c = static_cast<__nv_bfloat16 *>(c_kv);
    a.kv_len_old = kv_len_old;
    a.n_new = n_new;
    a.D = D_I;
    a.Dc = D_qk;
    a.Bsub = sub_block;
    a.L_max = L_max;
    a.err = device_error;
    return cuda_status(launch_append(a, B, static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_kv_minmax(const void *k_I, void *k_minmax, const int32_t *kv_len_old, int B,
                         int n_new, int D_I, int64_t L_max, int sub_block, int32_t *device_error,
                         void *stream) {
    if (!k_I || !k_minmax || !kv_len_old || B < 1 || n_new < 0 || L_max < 1)
        return LSA_ERR_INVALID_ARG;
    if (sub_block < 1 || sub_block > 4096) return LSA_ERR_INVALID_ARG;
    if (D_I != 64 && D_I != 128) return LSA_ERR_UNSUPPORTED;
    if (B > 65535 || L_max > 0x7FFFFFFFll) return LSA_ERR_UNSUPPORTED;
    if (misaligned(k_I, 16) || misaligned(k_minmax, 16) || misaligned(kv_len_old, 4) ||
        misaligned(device_error, 4))
        return LSA_ERR_INVALID_ARG;
    if (n_new == 0) return LSA_OK;
    AppendArgs a;
    memset(&a, 0, sizeof a);
    a.k = static_cast<__nv_bfloat16 *>(const_cast<void *>(k_I));
    a.k_minmax = static_cast<__nv_bfloat16 *>(k_minmax);
    a.kv_len_old = kv_len_old;
    a.n_new = n_new;
    a.D = D_I;
    a.Bsub = sub_block;
    a.L_max = L_max;
    a.err = device_error;
    return cuda_status(launch_minmax(a, B, static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_get_error(const void *ws, int32_t *device_code, void *stream) {
    if (!ws || !device_code) return LSA_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e);
    int32_t v = 0;
    e = cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    *device_code = v;
    return v ? LSA_ERR_DEVICE : LSA_OK;
}

}  // extern "C"
