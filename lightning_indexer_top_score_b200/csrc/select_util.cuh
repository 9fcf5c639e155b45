// select_util.cuh -- block-level helpers of the radix top-K (shared by the select kernels and the
// tcgen05 scorer, whose last CTA per row derives the row's threshold digit).
#pragma once

#include "lsa_internal.cuh"

namespace lsa {

// Largest bin b of hist[0..nbins) with suffix(b) = sum_{i >= b} hist[i] >= need (need >= 1,
// total >= need).  *gt = suffix(b + 1).  Every thread of the block must call it; results are
// valid for all threads on return.  scratch: >= 33 words of shared memory.
__device__ __forceinline__ void find_threshold(const uint32_t *hist, int nbins, uint32_t need, int *bin_out,
                               uint32_t *gt_out, uint32_t *scratch) {
    const int nthr = blockDim.x;
    const int per = (nbins + nthr - 1) / nthr;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
    const int lo = tid * per;
    const int hi = min(nbins, lo + per);
    uint32_t local = 0;
    for (int i = lo; i < hi; ++i) local += hist[i];
    // inclusive suffix sum over threads (higher thread index = higher bins)
    uint32_t v = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_down_sync(0xFFFFFFFFu, v, o);
        if (lane + o < 32) v += n;
    }
    if (lane == 0) scratch[warp] = v;  // warp total
    __syncthreads();
    uint32_t above = 0;
    for (int w2 = warp + 1; w2 < nwarps; ++w2) above += scratch[w2];
    const uint32_t incl = v + above;     // sum over threads >= tid
    const uint32_t excl = incl - local;  // sum over threads > tid
    if (excl < need && incl >= need) {
        uint32_t acc = excl;
        for (int i = hi - 1; i >= lo; --i) {
            if (acc + hist[i] >= need) {
                scratch[32] = (uint32_t)i;
                scratch[33] = acc;
                break;
            }
            acc += hist[i];
        }
    }
    __syncthreads();
    *bin_out = (int)scratch[32];
    *gt_out = scratch[33];
    __syncthreads();
}

// Block-wide sum; every thread gets the total.
__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t *scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    uint32_t tot = 0;
    for (int w2 = 0; w2 < nwarps; ++w2) tot += scratch[w2];
    __syncthreads();
    return tot;
}


// Threshold digit of a row from its full histogram (in shared memory): every thread gets
// thr (-1 when the row holds at most K candidates: all are taken), gt and total.
__device__ __forceinline__ void row_threshold(const uint32_t *hist, int K, int *thr, uint32_t *gt,
                                              uint32_t *total, uint32_t *scratch) {
    uint32_t loc = 0;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) loc += hist[i];
    *total = block_sum(loc, scratch);
    *thr = -1;
    *gt = 0;
    if (*total > (uint32_t)K) find_threshold(hist, kHistBins, (uint32_t)K, thr, gt, scratch);
}

}  // namespace lsa
