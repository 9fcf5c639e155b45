// append.cu -- KV-cache append and sub-block-mean upkeep for Hierarchical Indexing.
//
// Paper: Sec. 3.3 -- Hierarchical Indexing reads the sub-block mean keys k_mean from a
// per-sequence cache; Table 4's overhead list names their upkeep.  Each sub-block touched
// by an append is recomputed from its keys (those already cached and the appended ones): fp32
// sum of the present tokens in position order, divided by their count, rounded once to bf16.
// A partial last sub-block therefore always holds the mean of the tokens present so far,
// whatever the append history.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 128;

// One launch per call, grid (n_new + touched sub-blocks, B), 128 threads:
//   CTA x < n_new           copies new row x of k_I and/or c_kv (16 B per thread-step);
//   CTA x = n_new + j       recomputes the mean of the j-th sub-block the append touches, from
//                           the cache for the tokens before kv_len_old and from k_new for the
//                           new ones (so it does not wait for the copies), in position order.
__global__ void __launch_bounds__(kThreads) append_kernel(AppendArgs a) {
    const int64_t b = blockIdx.y, x = blockIdx.x;
    const int64_t old = a.kv_len_old[b];
    if (old < 0 || old + a.n_new > a.L_max) {
        if (x == 0 && threadIdx.x == 0) raise_error(a.err, LSA_DEVERR_APPEND);
        return;
    }
    if (x < a.n_new) {
        const int64_t pos = old + x;
        if (a.k_new) {
            const uint4 *src = reinterpret_cast<const uint4 *>(a.k_new + (b * a.n_new + x) * a.D);
            uint4 *dst = reinterpret_cast<uint4 *>(a.k + (b * a.L_max + pos) * a.D);
            for (int j = threadIdx.x; j < a.D / 8; j += blockDim.x) dst[j] = src[j];
        }
        if (a.c_new) {
            const uint4 *src = reinterpret_cast<const uint4 *>(a.c_new + (b * a.n_new + x) * a.Dc);
            uint4 *dst = reinterpret_cast<uint4 *>(a.c + (b * a.L_max + pos) * a.Dc);
            for (int j = threadIdx.x; j < a.Dc / 8; j += blockDim.x) dst[j] = src[j];
        }
        return;
    }
    if (!a.k_new || !a.k_mean) return;
    const int64_t len = old + a.n_new;
    const int64_t n = old / a.Bsub + (x - a.n_new);
    const int64_t lo = n * a.Bsub;
    if (lo >= len) return;
    const int64_t hi = lo + a.Bsub < len ? lo + a.Bsub : len;
    const __nv_bfloat16 *k = a.k + b * a.L_max * a.D;
    const __nv_bfloat16 *kn = a.k_new + b * a.n_new * a.D;
    const int64_t nb = (a.L_max + a.Bsub - 1) / a.Bsub;
    for (int d = threadIdx.x; d < a.D; d += blockDim.x) {
        float s = 0.f;
        for (int64_t p = lo; p < hi; ++p)
            s += __bfloat162float(p < old ? k[p * a.D + d] : kn[(p - old) * a.D + d]);
        a.k_mean[(b * nb + n) * a.D + d] = __float2bfloat16_rn(s / (float)(hi - lo));
    }
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
    const int touched = (a.k_new && a.k_mean) ? (a.n_new + a.Bsub - 1) / a.Bsub + 1 : 0;
    dim3 g((unsigned)(a.n_new + touched), (unsigned)B);
    append_kernel<<<g, kThreads, 0, s>>>(a);
    return launched();
}

}  // namespace lsa
