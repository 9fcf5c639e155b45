// append.cu -- KV-cache append and sub-block-mean upkeep for Hierarchical Indexing.
//
// Paper: Sec. 3.3 -- the sub-block mean keys k_mean are computed once for each sequence and
// kept in a cache; Table 4's overhead list names their maintenance.  Each sub-block touched
// by an append is recomputed from the key cache: fp32 sum of the present tokens in position
// order, divided by their count, rounded once to bf16.  A partial last sub-block therefore
// always holds the mean of the tokens present so far, whatever the append history.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kCopyThreads = 128;

// grid (n_new, B): copy one new row of k_I and/or c_kv (16 B per thread-step).
__global__ void __launch_bounds__(kCopyThreads) append_rows_kernel(AppendArgs a) {
    const int64_t b = blockIdx.y, i = blockIdx.x;
    const int64_t old = a.kv_len_old[b];
    if (old < 0 || old + a.n_new > a.L_max) {
        if (i == 0 && threadIdx.x == 0) raise_error(a.err, LSA_DEVERR_APPEND);
        return;
    }
    const int64_t pos = old + i;
    if (a.k_new) {
        const uint4 *src = reinterpret_cast<const uint4 *>(a.k_new + (b * a.n_new + i) * a.D);
        uint4 *dst = reinterpret_cast<uint4 *>(a.k + (b * a.L_max + pos) * a.D);
        for (int j = threadIdx.x; j < a.D / 8; j += blockDim.x) dst[j] = src[j];
    }
    if (a.c_new) {
        const uint4 *src = reinterpret_cast<const uint4 *>(a.c_new + (b * a.n_new + i) * a.Dc);
        uint4 *dst = reinterpret_cast<uint4 *>(a.c + (b * a.L_max + pos) * a.Dc);
        for (int j = threadIdx.x; j < a.Dc / 8; j += blockDim.x) dst[j] = src[j];
    }
}

// grid (touched sub-blocks, B), D threads: recompute the means of the touched sub-blocks.
__global__ void append_means_kernel(AppendArgs a) {
    const int64_t b = blockIdx.y;
    const int64_t old = a.kv_len_old[b];
    if (old < 0 || old + a.n_new > a.L_max) return;
    const int64_t len = old + a.n_new;
    const int64_t n = old / a.Bsub + blockIdx.x;
    const int64_t lo = n * a.Bsub;
    if (lo >= len) return;
    const int64_t hi = lo + a.Bsub < len ? lo + a.Bsub : len;
    const int d = threadIdx.x;
    if (d >= a.D) return;
    const __nv_bfloat16 *k = a.k + b * a.L_max * a.D;
    float s = 0.f;
    for (int64_t p = lo; p < hi; ++p) s += __bfloat162float(k[p * a.D + d]);
    const int64_t nb = (a.L_max + a.Bsub - 1) / a.Bsub;
    a.k_mean[(b * nb + n) * a.D + d] = __float2bfloat16_rn(s / (float)(hi - lo));
}

// grid (touched sub-blocks, B), D threads: recompute the MinMax rows of the touched sub-blocks
// (LongCat Sparse Attention, Sec. 5.3.5 pooling ablation): row n = (element-wise max,
// element-wise min) of the present tokens of sub-block n, both exact bf16 values of the cache.
__global__ void append_minmax_kernel(AppendArgs a) {
    const int64_t b = blockIdx.y;
    const int64_t old = a.kv_len_old[b];
    if (old < 0 || old + a.n_new > a.L_max) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(a.err, LSA_DEVERR_APPEND);
        return;
    }
    const int64_t len = old + a.n_new;
    const int64_t n = old / a.Bsub + blockIdx.x;
    const int64_t lo = n * a.Bsub;
    if (lo >= len) return;
    const int64_t hi = lo + a.Bsub < len ? lo + a.Bsub : len;
    const int d = threadIdx.x;
    if (d >= a.D) return;
    const __nv_bfloat16 *k = a.k + b * a.L_max * a.D;
    __nv_bfloat16 mx = k[lo * a.D + d], mn = mx;
    for (int64_t p = lo + 1; p < hi; ++p) {
        const __nv_bfloat16 v = k[p * a.D + d];
        mx = __hmax(mx, v);
        mn = __hmin(mn, v);
    }
    const int64_t nb = (a.L_max + a.Bsub - 1) / a.Bsub;
    __nv_bfloat16 *row = a.k_minmax + (b * nb + n) * 2 * a.D;
    row[d] = mx;
    row[a.D + d] = mn;
}

}  // namespace

cudaError_t launch_minmax(const AppendArgs &a, int B, cudaStream_t s) {
    if (B <= 0 || a.n_new <= 0) return cudaSuccess;
    const int touched = (a.n_new + a.Bsub - 1) / a.Bsub + 1;
    dim3 g((unsigned)touched, (unsigned)B);
    append_minmax_kernel<<<g, a.D, 0, s>>>(a);
    return launched();
}

cudaError_t launch_append(const AppendArgs &a, int B, cudaStream_t s) {
    if (B <= 0 || a.n_new <= 0) return cudaSuccess;
    dim3 g1((unsigned)a.n_new, (unsigned)B);
    append_rows_kernel<<<g1, kCopyThreads, 0, s>>>(a);
    cudaError_t e = launched();
    if (e != cudaSuccess || !a.k_new || !a.k_mean) return e;
    const int touched = (a.n_new + a.Bsub - 1) / a.Bsub + 1;
    dim3 g2((unsigned)touched, (unsigned)B);
    append_means_kernel<<<g2, a.D, 0, s>>>(a);
    return launched();
}

}  // namespace lsa
