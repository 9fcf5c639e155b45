// score_cc.cu -- Lightning Indexer scores on the CUDA cores (all three scoring modes).
//
// Paper: Sec. 2.2 Eq. 1  I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]);
//        Sec. 3.3 Eq. 9  page score = sum over the page's sub-block means of Eq. 1;
//        Sec. 3.3 Eq. 10 stage-2 token scores inside the recalled pages.
//
// One thread scores one unit (a token, a page, or a stage-2 slot).  The query's H x D
// indexer query is staged in shared memory transposed (qT[d][j], fp32) so that one 16-byte
// broadcast load feeds four heads' FMAs; the key row lives in registers.  fp32 accumulation.
// This is the general path (any H multiple of 8, D in {64, 128}); the decode stream on the
// tensor cores lives in score_tc.cu.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Eq. 1 for one key row held in registers.
template <int D>
__device__ __forceinline__ float score_key(const float *__restrict__ qT, const float *__restrict__ w,
                                           int H, const __nv_bfloat16 *__restrict__ key) {
    uint4 kr[D / 8];
    const uint4 *src = reinterpret_cast<const uint4 *>(key);
#pragma unroll
    for (int i = 0; i < D / 8; ++i) kr[i] = __ldg(src + i);
    float score = 0.f;
    for (int hc = 0; hc < H; hc += 8) {
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            const uint32_t wv[4] = {kr[i].x, kr[i].y, kr[i].z, kr[i].w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float kd = (e & 1) ? bf_hi(wv[e >> 1]) : bf_lo(wv[e >> 1]);
                const float4 qa = *reinterpret_cast<const float4 *>(qT + (i * 8 + e) * H + hc);
                const float4 qb = *reinterpret_cast<const float4 *>(qT + (i * 8 + e) * H + hc + 4);
                acc[0] = fmaf(qa.x, kd, acc[0]);
                acc[1] = fmaf(qa.y, kd, acc[1]);
                acc[2] = fmaf(qa.z, kd, acc[2]);
                acc[3] = fmaf(qa.w, kd, acc[3]);
                acc[4] = fmaf(qb.x, kd, acc[4]);
                acc[5] = fmaf(qb.y, kd, acc[5]);
                acc[6] = fmaf(qb.z, kd, acc[6]);
                acc[7] = fmaf(qb.w, kd, acc[7]);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) score = fmaf(w[hc + j], fmaxf(acc[j], 0.f), score);
    }
    return score;
}

template <int D>
__global__ void __launch_bounds__(kThreads) score_cc_kernel(ScoreArgs a, int64_t row0) {
    extern __shared__ __align__(16) float sm[];
    const int H = a.H;
    float *qT = sm;           // [D][H]
    float *wsm = sm + D * H;  // [H]

    const int64_t r = row0 + blockIdx.y;
    const int64_t b = r / a.T;
    const int64_t t = a.q_pos[r];
    const int64_t len = a.kv_len[b];
    if (!(t >= 0 && t < len && len <= a.L_max)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(a.err, LSA_DEVERR_QPOS);
        return;
    }
    const Regions g = regions_of(t, a.Ks, a.Kw);
    int64_t n_units = 0;
    if (a.mode == kScoreTokens) {
        n_units = g.dyn_hi - g.dyn_lo;
    } else if (a.mode == kScorePages) {
        n_units = (g.dyn_hi > g.dyn_lo) ? (g.dyn_hi - 1) / a.P - g.dyn_lo / a.P + 1 : 0;
    } else {
        n_units = (int64_t)a.page_count[r] * a.P;
    }
    const int64_t u0 = (int64_t)blockIdx.x * kThreads;
    if (u0 >= n_units) return;

    const __nv_bfloat16 *qr = a.q + r * H * D;
    for (int i = threadIdx.x; i < H * D; i += kThreads) {
        const int j = i / D, d = i - j * D;
        qT[d * H + j] = __bfloat162float(qr[i]);
    }
    for (int j = threadIdx.x; j < H; j += kThreads) wsm[j] = __bfloat162float(a.w[r * H + j]);
    __syncthreads();

    const int64_t u = u0 + threadIdx.x;
    if (u >= n_units) return;
    const __nv_bfloat16 *kseq = a.keys + b * a.key_seq_stride;
    float *out = a.out + r * a.out_stride;
    float score;
    if (a.mode == kScoreTokens) {
        const int64_t pos = g.dyn_lo + u;
        score = score_key<D>(qT, wsm, H, kseq + pos * D);
        out[pos] = score;
    } else if (a.mode == kScorePages) {
        const int64_t page = g.dyn_lo / a.P + u;
        const int per = a.P / a.Bsub;
        const int64_t nb = (len + a.Bsub - 1) / a.Bsub;
        int64_t n_lo = page * per, n_hi = n_lo + per;
        if (n_hi > nb) n_hi = nb;
        score = 0.f;
        for (int64_t n = n_lo; n < n_hi; ++n) score += score_key<D>(qT, wsm, H, kseq + n * D);
        out[page] = score;
    } else {
        const int64_t j = u / a.P, i = u - j * a.P;
        const int64_t pos = (int64_t)a.page_list[r * a.page_stride + j] * a.P + i;
        if (pos >= g.dyn_lo && pos < g.dyn_hi) {
            score = score_key<D>(qT, wsm, H, kseq + pos * D);
        } else {
            out[u] = excluded_score();
            return;
        }
        out[u] = score;
    }
    if (!isfinite(score)) raise_error(a.err, LSA_DEVERR_NONFINITE);
}

}  // namespace

cudaError_t launch_score(const ScoreArgs &a, int64_t rows, int64_t max_units, cudaStream_t s) {
    if (rows <= 0 || max_units <= 0) return cudaSuccess;
    const size_t smem = (size_t)(a.D * a.H + a.H) * sizeof(float);
    const int64_t gx = (max_units + kThreads - 1) / kThreads;
    if (gx > 0x7FFFFFFF) return cudaErrorInvalidValue;
    cudaError_t e;
    if (a.D == 128) {
        e = cudaFuncSetAttribute(score_cc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
    } else {
        e = cudaFuncSetAttribute(score_cc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
    }
    if (e != cudaSuccess) return e;
    for (int64_t r0 = 0; r0 < rows; r0 += 65535) {
        const int64_t nr = rows - r0 < 65535 ? rows - r0 : 65535;
        dim3 grid((unsigned)gx, (unsigned)nr);
        if (a.D == 128)
            score_cc_kernel<128><<<grid, kThreads, smem, s>>>(a, r0);
        else
            score_cc_kernel<64><<<grid, kThreads, smem, s>>>(a, r0);
        e = launched();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lsa
