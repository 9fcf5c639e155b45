// lsa_internal.cuh -- shared device helpers and launcher declarations of liblsa.so.
//
// Everything here is private to the library: the public boundary is include/lsa.h.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/lsa.h"

namespace lsa {

// ---------------------------------------------------------------- regions (Sec. 3.1)
// Streaming-aware split of query t (0-based): sink = [0, min(Ks, t+1)),
// swa = [max(Ks, t-Kw+1), t], dyn = [Ks, t-Kw].  Half-open bounds below.
struct Regions {
    int64_t sink_hi, swa_lo, swa_hi, dyn_lo, dyn_hi;
};

__host__ __device__ inline Regions regions_of(int64_t t, int Ks, int Kw) {
    Regions r;
    r.sink_hi = (t + 1 < Ks) ? t + 1 : Ks;
    r.swa_lo = t - Kw + 1;
    if (r.swa_lo < Ks) r.swa_lo = Ks;
    r.swa_hi = t + 1;
    if (r.swa_hi < r.swa_lo) r.swa_hi = r.swa_lo;
    r.dyn_lo = Ks;
    r.dyn_hi = t - Kw + 1;
    if (r.dyn_hi < r.dyn_lo) r.dyn_hi = r.dyn_lo;
    return r;
}

// ---------------------------------------------------------------- score ordering
// Monotone map float -> uint32 (larger float -> larger key).  The bit pattern
// 0xFFFFFFFF (a negative NaN no arithmetic produces here) maps to key 0 and marks a slot
// that takes no part in a selection.
constexpr uint32_t kExcludedBits = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 ranks as +0.0 (they are the same score)
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float excluded_score() { return __uint_as_float(kExcludedBits); }

// ---------------------------------------------------------------- device error word
__device__ __forceinline__ void raise_error(int32_t *err, int32_t bits) {
    if (err) atomicOr(err, bits);
}

// Checks the (kv_len, q_pos) pair of a query; raises LSA_DEVERR_QPOS when invalid.
__device__ __forceinline__ bool query_ok(int64_t t, int64_t len, int64_t L_max, int32_t *err) {
    bool ok = (t >= 0) && (t < len) && (len <= L_max);
    if (!ok) raise_error(err, LSA_DEVERR_QPOS);
    return ok;
}

// ---------------------------------------------------------------- selection arguments
// A selection row is one query's candidate list; slots are laid out in ascending position
// order, so "lower slot" == "lower position" for the tie-break.
enum SelectMode : int {
    kSelTokens = 0,  // slot = token position, range = dyn of the query
    kSelPages = 1,   // slot = page id, range = pages intersecting dyn
    kSelStage2 = 2,  // slot = j*P + i (i-th token of the j-th recalled page), range [0, n*P)
};

constexpr int kHistBits = 12;              // top digit of the 32-bit key
constexpr int kHistBins = 1 << kHistBits;  // 4096
constexpr int kMaxSelect = 4096;           // largest K (tokens) or M (pages)
// per-row selection counters: n_sure, n_cand, threshold digit, n_valid, scorer CTAs done
constexpr int kCountStride = 8;

struct SelectArgs {
    const float *scores;     // score row r at scores + r * row_stride
    int64_t row_stride;
    int mode;
    const int32_t *q_pos;    // [rows]
    const int32_t *kv_len;   // [B]
    int T;                   // queries per sequence (row r -> sequence r / T)
    int64_t L_max;
    int Ks, Kw, P;
    const int32_t *page_list;   // kSelStage2: [rows, page_stride] ascending page ids
    const int32_t *page_count;  // kSelStage2: [rows]
    int page_stride;
    int K;                   // how many to select
    uint32_t *hist;          // [rows, kHistBins]
    int32_t *counts;         // [rows, kCountStride]
    int thr_ready;           // counts[2..3] already hold the threshold (set by the scorer)
    int32_t *sure;           // [rows, sure_stride]
    int sure_stride;
    int32_t *cand;           // [rows, cand_stride]
    int64_t cand_stride;
    int32_t *out;            // [rows, out_stride] selected positions ascending, -1 padded
    int out_stride;
    int32_t *out_count;      // [rows] or nullptr
    int32_t *err;
};

// Row range [lo, hi) in slot units; false when the row is empty or invalid.
__device__ __forceinline__ bool select_row_range(const SelectArgs &a, int64_t r, int64_t &lo,
                                                 int64_t &hi) {
    lo = hi = 0;
    if (a.mode == kSelStage2) {
        hi = (int64_t)a.page_count[r] * a.P;
        return hi > 0;
    }
    int64_t t = a.q_pos[r];
    int64_t len = a.kv_len[r / a.T];
    if (!(t >= 0 && t < len && len <= a.L_max)) return false;  // flagged by the scorer
    Regions g = regions_of(t, a.Ks, a.Kw);
    if (g.dyn_hi <= g.dyn_lo) return false;
    if (a.mode == kSelTokens) {
        lo = g.dyn_lo;
        hi = g.dyn_hi;
    } else {
        lo = g.dyn_lo / a.P;
        hi = (g.dyn_hi - 1) / a.P + 1;
    }
    return true;
}

__device__ __forceinline__ int64_t slot_to_pos(const SelectArgs &a, int64_t r, int64_t slot) {
    if (a.mode != kSelStage2) return slot;
    int64_t pg = a.page_list[r * a.page_stride + slot / a.P];
    return pg * a.P + slot % a.P;
}

// ---------------------------------------------------------------- scoring arguments
enum ScoreMode : int {
    kScoreTokens = 0,  // unit = token of dyn; out[r * out_stride + pos]
    kScorePages = 1,   // unit = page intersecting dyn; out[r * out_stride + page] = Eq. 9
    kScoreStage2 = 2,  // unit = slot j*P + i of the recalled pages; out[r * out_stride + slot]
};

struct ScoreArgs {
    const __nv_bfloat16 *q;     // [rows, H, D]
    const __nv_bfloat16 *w;     // [rows, H]
    const __nv_bfloat16 *keys;  // k_I [B, L_max, D] or k_mean [B, NB, D]
    int64_t key_seq_stride;     // elements between sequences of `keys`
    const int32_t *q_pos;
    const int32_t *kv_len;
    int T, H, D;
    int64_t L_max;
    int Ks, Kw;
    int P, Bsub;                // page, sub-block (pages / stage 2)
    const int32_t *page_list;   // stage 2
    const int32_t *page_count;  // stage 2
    int page_stride;
    int mode;
    int minmax;                 // pages mode: keys are MinMax rows (k_max | k_min) of 2 D dims
    float *out;
    int64_t out_stride;
    int32_t *err;
};

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error; all run on `s`.
cudaError_t launch_score(const ScoreArgs &a, int64_t rows, int64_t max_units, cudaStream_t s);
// True when launch_select resolves these rows in one launch (no histogram or counters used).
bool select_is_small(int64_t rows, int64_t max_slots);
// Zero the row histograms and counters (needed before a scorer that fills the histogram).
cudaError_t select_clear(const SelectArgs &a, int64_t rows, cudaStream_t s);
// hist_ready: the histogram of the rows was already accumulated by the scoring kernel.
cudaError_t launch_select(const SelectArgs &a, int64_t rows, int64_t max_slots, cudaStream_t s,
                          bool hist_ready = false);

struct AttendArgs {
    const __nv_bfloat16 *q;     // [rows, H, 576]
    const __nv_bfloat16 *c;     // [B, L_max, 576]
    const int32_t *idx;         // [rows, K]
    const int32_t *q_pos;
    const int32_t *kv_len;
    int T, H, K;
    int64_t L_max;
    int Ks, Kw;
    float scale_log2;           // scale * log2(e)
    __nv_bfloat16 *out;         // [rows, H, 512]
    float *lse;                 // [rows, H]
    float *part_o;              // [rows, H, n_split, 512]
    float *part_lse;            // [rows, H, n_split]
    int n_split;
    int tiles_per_split;
    int use_tc;                 // 1: tcgen05 kernel (H == 128), 0: mma.sync kernel
    int32_t *err;
};

cudaError_t launch_attend(const AttendArgs &a, int64_t rows, cudaStream_t s);
cudaError_t launch_attend_tc(const AttendArgs &a, int64_t rows, cudaStream_t s);
int attend_tc_tile();           // keys per tile of the tcgen05 kernel
int attend_heads_per_cta(int H);  // heads per CTA of the mma.sync kernel

struct AppendArgs {
    const __nv_bfloat16 *k_new;  // [B, n_new, D]
    __nv_bfloat16 *k;            // [B, L_max, D]
    __nv_bfloat16 *k_mean;       // [B, NB, D]
    __nv_bfloat16 *k_minmax;     // [B, NB, 2 D] MinMax rows (k_max | k_min)
    const __nv_bfloat16 *c_new;  // [B, n_new, Dc]
    __nv_bfloat16 *c;            // [B, L_max, Dc]
    const int32_t *kv_len_old;
    int n_new, D, Dc, Bsub;
    int64_t L_max;
    int32_t *err;
};

cudaError_t launch_append(const AppendArgs &a, int B, cudaStream_t s);
// Refresh the MinMax rows of the sub-blocks that tokens [kv_len_old, kv_len_old + n_new) touch,
// from the keys already in the cache.
cudaError_t launch_minmax(const AppendArgs &a, int B, cudaStream_t s);

// Backward of the attention (attend_bwd.cu).
struct BwdArgs {
    const __nv_bfloat16 *q;     // [rows, H, 576]
    const __nv_bfloat16 *c;     // [B, L_max, 576]
    const int32_t *idx;         // [rows, K]
    const int32_t *kv_len;
    const int32_t *q_pos;
    const __nv_bfloat16 *dout;  // [rows, H, 512]
    const __nv_bfloat16 *o;     // [rows, H, 512] forward output, or null (with lse)
    const float *lse;           // [rows, H] forward lse (natural log), or null: recomputed
    float *dq;                  // [rows, H, 576] out
    float *dc;                  // [B, L_max, 576] accumulated
    int T, H, K, Ks, Kw;
    int64_t L_max;
    float scale;
    int32_t *err;
};

// Position of entry v of a query's virtual key list [sink | window | gathered picks] (the
// forward's order), or -1 past its end.  The picks must be ascending positions inside the dyn
// region; anything else raises LSA_DEVERR_INDEX and is skipped.
__device__ __forceinline__ int64_t bwd_key_pos(int32_t *err, const int32_t *idx, const Regions &g,
                                               int64_t n_sp, int64_t v) {
    const int64_t n_sink = g.sink_hi, n_swa = g.swa_hi - g.swa_lo;
    if (v < n_sink) return v;
    v -= n_sink;
    if (v < n_swa) return g.swa_lo + v;
    v -= n_swa;
    if (v >= n_sp) return -1;
    const int64_t p = idx[v];
    if (p >= g.dyn_lo && p < g.dyn_hi && (v == 0 || idx[v - 1] < p)) return p;
    raise_error(err, LSA_DEVERR_INDEX);
    return -1;
}

cudaError_t launch_attend_bwd(const BwdArgs &a, int64_t rows, cudaStream_t s);
// The tcgen05 backward: 64 heads per CTA, the forward's out and lse required.
bool attend_bwd_tc_supported(const BwdArgs &a);
cudaError_t launch_attend_bwd_tc(const BwdArgs &a, int64_t rows, cudaStream_t s);

// Called right after each kernel launch of this library: counts the launch (lsa_launch_count)
// and returns the launch's error state (cudaGetLastError).
cudaError_t launched();

}  // namespace lsa
