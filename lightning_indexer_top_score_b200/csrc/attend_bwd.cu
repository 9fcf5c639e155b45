// attend_bwd.cu -- backward of the Hybrid Sparse Attention over absorbed-MLA latent rows.
//
// Paper: Sec. 2.2 (u_t = Attn over the latent rows c_s, s in S_t), Sec. 3.1 (S_t = sink U swa
// U S_sparse), Sec. 4.1.1 (HFA backward: gather for dQ, scatter-add of the row gradients; the
// window halves the scattered set), Table 2 (the training setting).  With z_s = scale q.c_s,
// p_s = exp(z_s - lse), dp_s = dout . c_s[0:Dv], D = sum_s p_s dp_s and dz_s = p_s (dp_s - D):
//   dq   = scale sum_s dz_s c_s
//   dc_s += scale dz_s q + p_s dout   (the second term on the first Dv dims)
//
// One CTA per (query row, group of 16 heads), 512 threads, over the row's virtual key list
// [sink | window | gathered] in tiles of 32 rows (the forward's order).  Two passes:
//   pass 1 recomputes each head's lse and D exactly (online max / sums in fp32), so the backward
//          needs no forward output;
//   pass 2 forms P and dZ for the 16 x 32 (head, key) pairs of a tile, then dq += dZ K (each
//          thread owns 18 of a head's 576 dims) and the tile's row gradients dZ^T Q + P^T dO
//          (each thread owns 36 dims of one key), added once per CTA to the fp32 gradient
//          buffer with vector atomics.
// The contractions are small (16 heads per CTA), so they run on the CUDA cores in fp32 from the
// bf16 inputs; key tiles are double-buffered through cp.async with rows padded to 1168 bytes
// (16-byte reads by 8 consecutive lanes hit distinct bank groups).
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int HG = 16;          // heads per CTA
constexpr int NK = 32;          // keys per tile
constexpr int SROW = DQK + 8;   // padded K row (bf16 elements): 1168 B
constexpr int kThreads = 512;   // 16 warps; warp h <-> head h of the group in the pair phases
constexpr float kLog2e = 1.4426950408889634f;

struct Smem {
    __nv_bfloat16 q[HG][DQK];
    __nv_bfloat16 dout[HG][DV];
    __nv_bfloat16 k[2][NK][SROW];
    float p[HG][NK];
    float dz[HG][NK];
    int32_t pos[2][NK];
};

__device__ __forceinline__ int64_t bwd_key_pos(const BwdArgs &a, int64_t r, const Regions &g,
                                               int64_t n_sp, int64_t v) {
    const int64_t n_sink = g.sink_hi, n_swa = g.swa_hi - g.swa_lo;
    if (v < n_sink) return v;
    v -= n_sink;
    if (v < n_swa) return g.swa_lo + v;
    v -= n_swa;
    if (v >= n_sp) return -1;
    const int32_t *idx = a.idx + r * a.K;
    const int64_t p = idx[v];
    if (p >= g.dyn_lo && p < g.dyn_hi && (v == 0 || idx[v - 1] < p)) return p;
    raise_error(a.err, LSA_DEVERR_INDEX);
    return -1;
}

__device__ __forceinline__ void cp16(void *dst, const void *src, int bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src), "r"(bytes)
                 : "memory");
}

// Issues the copies of tile `tile` into stage st (all threads) and records its positions.
__device__ __forceinline__ void load_tile(Smem &S, int st, const BwdArgs &a, int64_t r, int64_t b,
                                          const Regions &g, int64_t n_sp, int64_t tile) {
    const int tid = threadIdx.x;
    if (tid < NK) S.pos[st][tid] = (int32_t)bwd_key_pos(a, r, g, n_sp, tile * NK + tid);
    __syncthreads();  // positions visible to every copying thread
    const __nv_bfloat16 *cseq = a.c + b * a.L_max * DQK;
    for (int e = tid; e < NK * (DQK / 8); e += kThreads) {
        const int j = e / (DQK / 8), pc = e - j * (DQK / 8);
        const int64_t pos = S.pos[st][j];
        cp16(&S.k[st][j][pc * 8], pos >= 0 ? cseq + pos * DQK + pc * 8 : cseq, pos >= 0 ? 16 : 0);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// s = q_h . c_j over DQK dims and dp = dout_h . c_j over DV dims (16-byte reads)
__device__ __forceinline__ void dots(const Smem &S, int st, int h, int j, float &s, float &dp) {
    float s0 = 0.f, s1 = 0.f, g0 = 0.f, g1 = 0.f;
    const uint4 *cr = reinterpret_cast<const uint4 *>(&S.k[st][j][0]);
    const uint4 *qr = reinterpret_cast<const uint4 *>(&S.q[h][0]);
    const uint4 *dr = reinterpret_cast<const uint4 *>(&S.dout[h][0]);
#pragma unroll 4
    for (int u = 0; u < DQK / 8; ++u) {
        const uint4 cv = cr[u], qv = qr[u];
        const __nv_bfloat162 *c2 = reinterpret_cast<const __nv_bfloat162 *>(&cv);
        const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 cf = __bfloat1622float2(c2[e]), qf = __bfloat1622float2(q2[e]);
            s0 = fmaf(qf.x, cf.x, s0);
            s1 = fmaf(qf.y, cf.y, s1);
        }
        if (u < DV / 8) {
            const uint4 dv = dr[u];
            const __nv_bfloat162 *d2 = reinterpret_cast<const __nv_bfloat162 *>(&dv);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 cf = __bfloat1622float2(c2[e]), df = __bfloat1622float2(d2[e]);
                g0 = fmaf(df.x, cf.x, g0);
                g1 = fmaf(df.y, cf.y, g1);
            }
        }
    }
    s = s0 + s1;
    dp = g0 + g1;
}

__global__ void __launch_bounds__(kThreads) hfa_bwd_kernel(BwdArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t r = blockIdx.x;
    const int h0 = blockIdx.y * HG;
    const int64_t b = r / a.T;
    const int64_t t = a.q_pos[r];
    const int64_t len = a.kv_len[b];
    if (!(t >= 0 && t < len && len <= a.L_max)) {
        if (tid == 0 && blockIdx.y == 0) raise_error(a.err, LSA_DEVERR_QPOS);
        return;
    }
    const Regions g = regions_of(t, a.Ks, a.Kw);
    // gathered picks of this row: the selection writes them ascending, -1 after the last
    __shared__ int nsp_s;
    if (tid == 0) nsp_s = 0;
    __syncthreads();
    {
        int c = 0;
        for (int i = tid; i < a.K; i += kThreads) c += (a.idx[r * a.K + i] >= 0);
        if (c) atomicAdd(&nsp_s, c);
    }
    // this row's q and dout for the 16 heads of the group
    {
        const uint4 *qg = reinterpret_cast<const uint4 *>(a.q + (r * a.H + h0) * (int64_t)DQK);
        for (int e = tid; e < HG * DQK / 8; e += kThreads)
            reinterpret_cast<uint4 *>(&S.q[0][0])[e] = qg[e];
        const uint4 *dg = reinterpret_cast<const uint4 *>(a.dout + (r * a.H + h0) * (int64_t)DV);
        for (int e = tid; e < HG * DV / 8; e += kThreads)
            reinterpret_cast<uint4 *>(&S.dout[0][0])[e] = dg[e];
    }
    __syncthreads();
    const int64_t n_sp = nsp_s;
    const int64_t n_total = g.sink_hi + (g.swa_hi - g.swa_lo) + n_sp;
    const int64_t n_tiles = (n_total + NK - 1) / NK;
    const float sl2 = a.scale * kLog2e;

    // ---------------- pass 1: lse and D per head (warp h, lane j = key of the tile)
    const int h = warp, j = lane;
    float m = -INFINITY, l = 0.f, gsum = 0.f;  // uniform across warp h after each tile
    if (n_tiles > 0) load_tile(S, 0, a, r, b, g, n_sp, 0);
    for (int64_t it = 0; it < n_tiles; ++it) {
        const int st = (int)(it & 1);
        if (it + 1 < n_tiles) {
            load_tile(S, st ^ 1, a, r, b, g, n_sp, it + 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        float s, dp;
        dots(S, st, h, j, s, dp);
        const bool valid = S.pos[st][j] >= 0;
        const float z = valid ? s * sl2 : -INFINITY;  // log2 units
        float mt = z;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, o));
        const float mn = fmaxf(m, mt);
        float e = (valid && mn > -INFINITY) ? exp2f(z - mn) : 0.f;
        float ed = e * dp;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            e += __shfl_xor_sync(0xFFFFFFFFu, e, o);
            ed += __shfl_xor_sync(0xFFFFFFFFu, ed, o);
        }
        const float alpha = (m > -INFINITY) ? exp2f(m - mn) : 0.f;
        l = l * alpha + e;
        gsum = gsum * alpha + ed;
        m = mn;
        __syncthreads();  // the stage is refilled by the next iteration's copies
    }
    const float lse2 = (l > 0.f) ? m + log2f(l) : INFINITY;  // exp2(z - lse2) = p; no keys: p = 0
    const float D = (l > 0.f) ? gsum / l : 0.f;
    if (!isfinite(l) || !isfinite(gsum)) raise_error(a.err, LSA_DEVERR_NONFINITE);

    // ---------------- pass 2: dq and the row gradients
    float dq[18];  // thread (h, lane) owns dims 2 lane + 64 k, +1  (k < 9)
#pragma unroll
    for (int k = 0; k < 18; ++k) dq[k] = 0.f;
    const int jc = tid >> 4;        // key of the tile in the row-gradient phase
    const int dl = (tid & 15) * 2;  // first dim pair: dims dl + 32 k, +1  (k < 18)
    float *dc_seq = a.dc + b * a.L_max * DQK;
    if (n_tiles > 0) load_tile(S, 0, a, r, b, g, n_sp, 0);
    for (int64_t it = 0; it < n_tiles; ++it) {
        const int st = (int)(it & 1);
        if (it + 1 < n_tiles) {
            load_tile(S, st ^ 1, a, r, b, g, n_sp, it + 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        {
            float s, dp;
            dots(S, st, h, j, s, dp);
            const bool valid = S.pos[st][j] >= 0;
            const float p = valid ? exp2f(s * sl2 - lse2) : 0.f;
            S.p[h][j] = p;
            S.dz[h][j] = p * (dp - D) * a.scale;
        }
        __syncthreads();
        // dq[h] += sum_j dz[h][j] c_j
#pragma unroll 4
        for (int jj = 0; jj < NK; ++jj) {
            const float w = S.dz[h][jj];
            const __nv_bfloat162 *cr = reinterpret_cast<const __nv_bfloat162 *>(&S.k[st][jj][0]);
#pragma unroll
            for (int k = 0; k < 9; ++k) {
                const float2 cf = __bfloat1622float2(cr[lane + 32 * k]);
                dq[2 * k] = fmaf(w, cf.x, dq[2 * k]);
                dq[2 * k + 1] = fmaf(w, cf.y, dq[2 * k + 1]);
            }
        }
        // row gradient of key jc: sum_h dz[h][jc] q_h + p[h][jc] dout_h (first DV dims)
        {
            float acc[36];
#pragma unroll
            for (int k = 0; k < 36; ++k) acc[k] = 0.f;
#pragma unroll 2
            for (int hh = 0; hh < HG; ++hh) {
                const float wz = S.dz[hh][jc], wp = S.p[hh][jc];
                const __nv_bfloat162 *qr = reinterpret_cast<const __nv_bfloat162 *>(&S.q[hh][0]);
                const __nv_bfloat162 *dr = reinterpret_cast<const __nv_bfloat162 *>(&S.dout[hh][0]);
#pragma unroll
                for (int k = 0; k < 18; ++k) {
                    const int d2 = (dl >> 1) + 16 * k;  // bf16-pair index of dims dl + 32 k
                    const float2 qf = __bfloat1622float2(qr[d2]);
                    acc[2 * k] = fmaf(wz, qf.x, acc[2 * k]);
                    acc[2 * k + 1] = fmaf(wz, qf.y, acc[2 * k + 1]);
                    if (dl + 32 * k < DV) {
                        const float2 df = __bfloat1622float2(dr[d2]);
                        acc[2 * k] = fmaf(wp, df.x, acc[2 * k]);
                        acc[2 * k + 1] = fmaf(wp, df.y, acc[2 * k + 1]);
                    }
                }
            }
            const int64_t pos = S.pos[st][jc];
            if (pos >= 0) {
                float *row = dc_seq + pos * DQK + dl;
#pragma unroll
                for (int k = 0; k < 18; ++k)
                    atomicAdd(reinterpret_cast<float2 *>(row + 32 * k),
                              make_float2(acc[2 * k], acc[2 * k + 1]));
            }
        }
        __syncthreads();  // p / dz and the stage are reused by the next tile
    }
    float *dqo = a.dq + (r * a.H + h0 + h) * (int64_t)DQK;
#pragma unroll
    for (int k = 0; k < 9; ++k)
        *reinterpret_cast<float2 *>(dqo + 2 * lane + 64 * k) = make_float2(dq[2 * k], dq[2 * k + 1]);
}

}  // namespace

cudaError_t launch_attend_bwd(const BwdArgs &a, int64_t rows, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    if (rows > 0x7FFFFFFF || a.H % HG) return cudaErrorInvalidValue;
    const int smem = (int)sizeof(Smem);
    cudaError_t e = cudaFuncSetAttribute(hfa_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)rows, (unsigned)(a.H / HG));
    hfa_bwd_kernel<<<grid, kThreads, smem, s>>>(a);
    return launched();
}

}  // namespace lsa
