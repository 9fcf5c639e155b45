// score_tc.cuh -- arguments and launcher of the tcgen05 scoring kernel (score_tc.cu).
#pragma once

#include <cuda.h>

#include "lsa_internal.cuh"

namespace lsa {

struct TcScoreArgs {
    const __nv_bfloat16 *q;     // [rows, H, D]
    // FP8 indexer (tokens mode only): E4M3 query codes [rows, H, D] with scales [rows, H],
    // key scales [B, L_max]; the keys are E4M3 codes [B * L_max, D]
    const uint8_t *q8;
    const float *qscale;
    const float *kscale;
    const __nv_bfloat16 *w;     // [rows, H]
    const int32_t *q_pos;
    const int32_t *kv_len;
    int T, H;
    int64_t L_max;
    int64_t nb_max;             // sub-blocks per sequence in the mean cache (pages mode)
    int Ks, Kw;
    int P, Bsub;
    int mode;                   // ScoreMode
    const int32_t *page_list;   // stage 2: [rows, page_stride]
    const int32_t *page_count;  // stage 2: [rows]
    int page_stride;
    float *out;
    int64_t out_stride;
    uint32_t *hist;             // [rows, kHistBins], zeroed before the launch; null: no histogram,
                                // no threshold step (the one-launch select needs neither)
    int32_t *counts;            // [rows, kCountStride], zeroed before the launch
    int sel_K;                  // how many the selection of this pass keeps
    int minmax;                 // pages mode only: keys are MinMax rows (k_max | k_min), 2 D wide
    int32_t *err;
    int chunk_tiles;            // set by the launcher
    int n_chunks;
};

// 2-D bf16 tensor map over [rows, inner] (row stride inner*2 bytes), box {box_inner, box_rows},
// SWIZZLE_128B.  False if the driver entry point is unavailable or the encoding is refused.
bool make_tmap_2d_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                       uint32_t box_inner, uint32_t box_rows);

// 2-D byte tensor map over [rows, inner] (row stride inner bytes), box {box_inner, box_rows},
// SWIZZLE_128B.
bool make_tmap_2d_u8(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                     uint32_t box_inner, uint32_t box_rows);

// FP8 scoring pass (tokens mode, D = 128, H in {64, 128}): keys8 are E4M3 codes [key_rows, D].
cudaError_t launch_score_tc_fp8(const TcScoreArgs &a, const void *keys8, int64_t key_rows, int D,
                                int64_t rows, int64_t max_tiles, cudaStream_t s);

// Whether the tensor-core path handles this shape (else the CUDA-core path is used).
bool tc_score_supported(int H, int D, int mode, int P, int Bsub, int64_t key_rows);

// keys: the key tensor viewed as [key_rows, D] bf16 (k_I: B*L_max rows, k_mean: B*nb_max rows).
// max_tiles: upper bound of 128-unit tiles per row.
cudaError_t launch_score_tc(const TcScoreArgs &a, const void *keys, int64_t key_rows, int D,
                            int64_t rows, int64_t max_tiles, cudaStream_t s);

// Multi-query scorer (score_mq.cu): token scoring (flat) or sub-block-mean page scoring (HI stage
// 1) of T >= 2 queries per sequence, G consecutive queries per CTA (G x H_I = 256 accumulator
// columns).
bool mq_score_supported(int H, int D, int T, int mode, int P, int Bsub, int minmax);
// B sequences of a.T queries each; keys: the key cache viewed as [key_rows, 128] bf16.
cudaError_t launch_score_mq(const TcScoreArgs &a, const void *keys, int64_t key_rows, int B,
                            int64_t max_tiles, cudaStream_t s);

}  // namespace lsa
