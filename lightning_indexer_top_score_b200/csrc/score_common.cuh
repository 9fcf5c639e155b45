// score_common.cuh -- pieces shared by the tensor-core scoring kernels (score_tc.cu,
// score_mq.cu): the CTA-level histogram of the selection's first digit and the per-row "last
// scoring CTA derives the threshold" step.
#pragma once

#include "lsa_internal.cuh"
#include "score_tc.cuh"
#include "select_util.cuh"

namespace lsa {

// Warp-collective: adds each lane's key to the CTA's histogram of top-12-bit digits (key 0 = none).
// Scores crowd into a few bins, so lanes with the same digit are merged first (one shared-memory
// atomic per distinct digit and warp instead of up to 32 on one address).
__device__ __forceinline__ void hist_add_warp(uint32_t *hist_s, uint32_t key) {
    const uint32_t bin = key ? (key >> (32 - kHistBits)) : 0xFFFFFFFFu;
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bin);
    if (bin != 0xFFFFFFFFu && (threadIdx.x & 31) == (uint32_t)(__ffs(peers) - 1))
        atomicAdd(&hist_s[bin], (uint32_t)__popc(peers));
}

// Called by every CTA of row r once its histogram contribution is flushed: the last one to
// finish (atomic count, no waiting) derives the row's threshold digit for the selection.
__device__ __forceinline__ void row_done(const TcScoreArgs &a, int64_t r, uint32_t *hist_s,
                                         uint32_t *scratch, int *s_last) {
    __threadfence();
    __syncthreads();
    int32_t *cnt = a.counts + r * kCountStride;
    if (threadIdx.x == 0) *s_last = (atomicAdd(&cnt[4], 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (*s_last) {
        __threadfence();
        const uint32_t *gh = a.hist + r * kHistBins;
        for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist_s[i] = __ldcg(gh + i);
        __syncthreads();
        int thr;
        uint32_t gt, total;
        row_threshold(hist_s, a.sel_K, &thr, &gt, &total, scratch);
        if (threadIdx.x == 0) {
            cnt[2] = thr;
            cnt[3] = (int32_t)total;
        }
    }
}

}  // namespace lsa
