// attend.cu -- Hybrid Sparse Attention (HFA) forward over absorbed-MLA latent rows.
//
// Paper: Sec. 2.2 (u_t = Attn over the latent rows c_s, s in S_t), Sec. 3.1 (S_t = sink U swa
// U S_sparse; the fixed tokens still take part in the normalisation, Fig. 1), Sec. 4.1.1 (HFA:
// the contiguous branch and the gathered branch are computed apart and merged by online-softmax
// rescaling).  Here both branches stream through the same pipeline: the key list of a query is
// the virtual sequence [sink rows | window rows | gathered rows], cut into 32-row tiles; a CTA
// owns one query, one group of up to 64 heads and one contiguous range of tiles (a split), keeps
// a running (max, sum) per head, and the splits are merged by the log-sum-exp rescaling of the
// paper in a second small kernel.  The tensor-core path is mma.sync m16n8k16 bf16 with fp32
// accumulation: S = Q K^T over all 576 latent dims, P = exp(S - m) in bf16, O += P V over the
// first 512 dims.
//
// Warp layout (2 warps per 16-head m-tile): warp (m, half) computes S for keys
// [16*half, 16*half+16) of the tile and accumulates O for value dims [256*half, 256*half+256).
// The two warps of an m-tile exchange row maxima and the bf16 P tile through shared memory
// (named barrier per pair).
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int SROW = DQK + 8;  // smem row stride in bf16 (1168 B: ldmatrix conflict-free)
constexpr int NK = 32;         // keys per tile
constexpr int STAGES = 3;
constexpr int PROW = NK + 8;   // P tile row stride (80 B)

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void pair_barrier(int id) {
    asm volatile("bar.sync %0, 64;\n" ::"r"(id));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

struct RowList {
    int64_t n_sink, n_swa, swa_lo, n_sp, dyn_lo, dyn_hi;
    const int32_t *idx;
};

// Position of virtual key v of the query (sink | window | gathered); -1 if none or invalid.
__device__ __forceinline__ int64_t vpos(const RowList &L, int64_t v, bool check, int32_t *err) {
    if (v < L.n_sink) return v;
    v -= L.n_sink;
    if (v < L.n_swa) return L.swa_lo + v;
    v -= L.n_swa;
    if (v >= L.n_sp) return -1;
    const int64_t p = L.idx[v];
    const bool ok = p >= L.dyn_lo && p < L.dyn_hi && (v == 0 || L.idx[v - 1] < p);
    if (!ok) {
        if (check) raise_error(err, LSA_DEVERR_INDEX);
        return -1;
    }
    return p;
}

template <int NM>
__global__ void __launch_bounds__(64 * NM, 1) hfa_kernel(AttendArgs a) {
    constexpr int NW = 2 * NM;
    constexpr int NT = 32 * NW;
    constexpr int HG = 16 * NM;
    extern __shared__ __align__(128) uint8_t smem[];
    __nv_bfloat16 *Qs = reinterpret_cast<__nv_bfloat16 *>(smem);
    __nv_bfloat16 *KVs = Qs + HG * SROW;
    __nv_bfloat16 *Ps = KVs + STAGES * NK * SROW;
    float *red = reinterpret_cast<float *>(Ps + 2 * NM * 16 * PROW);  // [2][NM][2][16]
    int *tile_ok = reinterpret_cast<int *>(red + 2 * NM * 2 * 16);   // [STAGES][NK]
    int *misc = tile_ok + STAGES * NK;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m = warp >> 1, half = warp & 1;
    const int64_t r = blockIdx.x;
    const int hg0 = blockIdx.y * HG;
    const int split = blockIdx.z;
    const int64_t b = r / a.T;
    const int64_t t = a.q_pos[r];
    const int64_t len = a.kv_len[b];
    const int H = a.H;
    const bool qok = (t >= 0 && t < len && len <= a.L_max);
    if (!qok) {
        if (tid == 0 && blockIdx.y == 0 && split == 0) raise_error(a.err, LSA_DEVERR_QPOS);
        return;
    }
    const Regions g = regions_of(t, a.Ks, a.Kw);
    RowList L;
    L.n_sink = g.sink_hi;
    L.n_swa = g.swa_hi - g.swa_lo;
    L.swa_lo = g.swa_lo;
    L.dyn_lo = g.dyn_lo;
    L.dyn_hi = g.dyn_hi;
    L.idx = a.idx + r * a.K;
    if (tid == 0) misc[0] = 0;
    __syncthreads();
    {
        int c = 0;
        for (int i = tid; i < a.K; i += NT) c += (L.idx[i] >= 0);
        if (c) atomicAdd(&misc[0], c);
    }
    __syncthreads();
    L.n_sp = misc[0];
    const int64_t n_total = L.n_sink + L.n_swa + L.n_sp;
    const int64_t ntiles = (n_total + NK - 1) / NK;
    const int64_t t0 = (int64_t)split * a.tiles_per_split;
    int64_t t1 = t0 + a.tiles_per_split;
    if (t1 > ntiles) t1 = ntiles;

    const __nv_bfloat16 *cseq = a.c + b * a.L_max * DQK;
    // ---- Q rows of this head group (rows >= H zero-filled)
    {
        const __nv_bfloat16 *qr = a.q + (r * H + hg0) * (int64_t)DQK;
        for (int i = tid; i < HG * (DQK / 8); i += NT) {
            const int row = i / (DQK / 8), ch = i - row * (DQK / 8);
            const bool v = hg0 + row < H;
            cp_async16(Qs + row * SROW + ch * 8, v ? qr + row * DQK + ch * 8 : a.q, v ? 16 : 0);
        }
    }
    auto load_tile = [&](int64_t ti, int st) {
        __nv_bfloat16 *dst = KVs + st * NK * SROW;
        for (int i = tid; i < NK * (DQK / 8); i += NT) {
            const int row = i / (DQK / 8), ch = i - row * (DQK / 8);
            const int64_t p = vpos(L, ti * NK + row, ch == 0, a.err);
            if (ch == 0) tile_ok[st * NK + row] = (p >= 0);
            cp_async16(dst + row * SROW + ch * 8, p >= 0 ? cseq + p * DQK + ch * 8 : cseq,
                       p >= 0 ? 16 : 0);
        }
    };
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
        if (t0 + s < t1) load_tile(t0 + s, s);
        cp_async_commit();
    }

    float oacc[32][4];
#pragma unroll
    for (int i = 0; i < 32; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};

    const int g4 = lane >> 2, c4 = lane & 3;
    const int arow = (lane & 7) + ((lane >> 3) & 1) * 8, acol = (lane >> 4) * 8;
    const int brow = (lane & 7) + (lane >> 4) * 8, bcol = ((lane >> 3) & 1) * 8;
    const __nv_bfloat16 *Qm = Qs + (m * 16) * SROW;
    bool nonfinite = false;

    for (int64_t it = t0; it < t1; ++it) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();
        {
            const int64_t nt = it + STAGES - 1;
            if (nt < t1) load_tile(nt, (int)((nt - t0) % STAGES));
            cp_async_commit();
        }
        const int st = (int)((it - t0) % STAGES);
        const int par = (int)((it - t0) & 1);
        const __nv_bfloat16 *KV = KVs + st * NK * SROW;

        // ---- S = Q K^T for keys [16*half, 16*half + 16)
        float sacc[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll 4
        for (int k = 0; k < DQK / 16; ++k) {
            uint32_t af[4], bf[4];
            ldsm_x4(af, Qm + arow * SROW + k * 16 + acol);
            ldsm_x4(bf, KV + (half * 16 + brow) * SROW + k * 16 + bcol);
            mma_bf16(sacc[0], af, bf[0], bf[1]);
            mma_bf16(sacc[1], af, bf[2], bf[3]);
        }
        // ---- scale, mask, row max
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < 2; ++n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = half * 16 + n * 8 + 2 * c4 + (e & 1);
                float z = sacc[n][e] * a.scale_log2;
                nonfinite |= !isfinite(z);
                if (!tile_ok[st * NK + key]) z = -INFINITY;
                sacc[n][e] = z;
                mx[e >> 1] = fmaxf(mx[e >> 1], z);
            }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xFFFFFFFFu, mx[i], 1));
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xFFFFFFFFu, mx[i], 2));
        }
        float *redp = red + ((par * NM + m) * 2) * 16;
        if (c4 == 0) {
            redp[half * 16 + g4] = mx[0];
            redp[half * 16 + g4 + 8] = mx[1];
        }
        pair_barrier(1 + m);
        float ref[2], alpha[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float other = redp[(1 - half) * 16 + g4 + 8 * i];
            const float mnew = fmaxf(m_run[i], fmaxf(mx[i], other));
            ref[i] = (mnew == -INFINITY) ? 0.f : mnew;
            alpha[i] = exp2f(m_run[i] - ref[i]);
            m_run[i] = mnew;
        }
        // ---- P = exp2(z - m), own row sums, bf16 P tile to shared memory
        __nv_bfloat16 *Pm = Ps + (par * NM + m) * 16 * PROW;
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const float p0 = exp2f(sacc[n][0] - ref[0]);
            const float p1 = exp2f(sacc[n][1] - ref[0]);
            const float p2 = exp2f(sacc[n][2] - ref[1]);
            const float p3 = exp2f(sacc[n][3] - ref[1]);
            rs[0] += p0 + p1;
            rs[1] += p2 + p3;
            const int col = half * 16 + n * 8 + 2 * c4;
            *reinterpret_cast<uint32_t *>(Pm + g4 * PROW + col) = pack_bf16(p0, p1);
            *reinterpret_cast<uint32_t *>(Pm + (g4 + 8) * PROW + col) = pack_bf16(p2, p3);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            rs[i] += __shfl_xor_sync(0xFFFFFFFFu, rs[i], 1);
            rs[i] += __shfl_xor_sync(0xFFFFFFFFu, rs[i], 2);
            l_run[i] = l_run[i] * alpha[i] + rs[i];
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            oacc[i][0] *= alpha[0];
            oacc[i][1] *= alpha[0];
            oacc[i][2] *= alpha[1];
            oacc[i][3] *= alpha[1];
        }
        pair_barrier(1 + m);
        // ---- O += P V for value dims [256*half, 256*half + 256)
#pragma unroll
        for (int ks = 0; ks < NK / 16; ++ks) {
            uint32_t pa[4];
            ldsm_x4(pa, Pm + arow * PROW + ks * 16 + acol);
#pragma unroll
            for (int n2 = 0; n2 < 16; ++n2) {
                uint32_t vb[4];
                ldsm_x4_t(vb, KV + (ks * 16 + arow) * SROW + half * 256 + n2 * 16 + acol);
                mma_bf16(oacc[2 * n2], pa, vb[0], vb[1]);
                mma_bf16(oacc[2 * n2 + 1], pa, vb[2], vb[3]);
            }
        }
    }
    cp_async_wait<0>();
    if (nonfinite) raise_error(a.err, LSA_DEVERR_NONFINITE);

    // ---- combine the two halves' row sums
    float *redl = red;  // reuse parity-0 slot after the loop
    __syncthreads();
    if (c4 == 0) {
        redl[(m * 2 + half) * 16 + g4] = l_run[0];
        redl[(m * 2 + half) * 16 + g4 + 8] = l_run[1];
    }
    __syncthreads();
    float lsum[2], inv[2], lse_n[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        lsum[i] = redl[(m * 2 + 0) * 16 + g4 + 8 * i] + redl[(m * 2 + 1) * 16 + g4 + 8 * i];
        inv[i] = lsum[i] > 0.f ? 1.f / lsum[i] : 0.f;
        lse_n[i] = lsum[i] > 0.f ? (m_run[i] + log2f(lsum[i])) * 0.6931471805599453f : -INFINITY;
    }
    // ---- write
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int h = hg0 + m * 16 + g4 + 8 * i;
        if (h >= H) continue;
        if (a.n_split == 1) {
            __nv_bfloat16 *o = a.out + (r * H + h) * (int64_t)DV + half * 256;
#pragma unroll
            for (int n = 0; n < 32; ++n) {
                const int col = n * 8 + 2 * c4;
                *reinterpret_cast<uint32_t *>(o + col) =
                    pack_bf16(oacc[n][2 * i] * inv[i], oacc[n][2 * i + 1] * inv[i]);
            }
            if (half == 0 && c4 == 0) a.lse[r * H + h] = lse_n[i];
        } else {
            float *o = a.part_o + ((r * H + h) * a.n_split + split) * (int64_t)DV + half * 256;
#pragma unroll
            for (int n = 0; n < 32; ++n) {
                const int col = n * 8 + 2 * c4;
                *reinterpret_cast<float2 *>(o + col) =
                    make_float2(oacc[n][2 * i] * inv[i], oacc[n][2 * i + 1] * inv[i]);
            }
            if (half == 0 && c4 == 0) a.part_lse[(r * H + h) * a.n_split + split] = lse_n[i];
        }
    }
}

// Log-sum-exp merge of the splits (Sec. 4.1.1's rescaling):
//   lse = ln sum_s e^{lse_s},  out = sum_s e^{lse_s - lse} o_s.
// Two forms, by the number of splits:
//   few splits   one warp per (row, head), kCombineWarps per CTA: each lane merges 16 of the 512
//                dims, four full warp lines per split;
//   many splits  one warp per (row, head, quarter of the dims): each lane merges 4 dims, with the
//                loads of kCombineBatch splits in flight before any is accumulated (a warp
//                walking many splits would otherwise wait on one load round trip per split).
// Both sum the splits in order, so they give the same bits.
constexpr int kCombineWarps = 8;
constexpr int kCombineBatch = 8;
constexpr int kCombineSplitMin = 8;  // splits from which the quarter form runs

// the split weights' maximum and normaliser of one (row, head)
__device__ __forceinline__ void combine_weights(const float *pl, int ns, float *mx, float *wsum) {
    float m = -INFINITY;
    for (int s = 0; s < ns; ++s) m = fmaxf(m, pl[s]);
    float w = 0.f;
    for (int s = 0; s < ns; ++s) w += (pl[s] == -INFINITY) ? 0.f : __expf(pl[s] - m);
    *mx = m;
    *wsum = w;
}

template <bool QUARTERS>
__global__ void __launch_bounds__(32 * kCombineWarps) hfa_combine_kernel(AttendArgs a,
                                                                        int64_t n_rh) {
    constexpr int Q = QUARTERS ? 4 : 1;  // warps per (row, head)
    constexpr int KV = 4 / Q;            // float4 per lane per split
    const int64_t item = (int64_t)blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
    if (item >= n_rh * Q) return;
    const int64_t rh = item / Q;  // row*H + head
    const int qd = (int)(item % Q);
    const int lane = threadIdx.x & 31;
    const int ns = a.n_split;
    const float *pl = a.part_lse + rh * ns;
    float mx, wsum;
    combine_weights(pl, ns, &mx, &wsum);
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    // lane's dims 4 (lane + 32 (qd KV + k)) .. + 3, k < KV, of every split
    const float4 *src = reinterpret_cast<const float4 *>(a.part_o + rh * ns * (int64_t)DV) +
                        32 * qd * KV + lane;
    constexpr int B = QUARTERS ? kCombineBatch : 1;
    float4 acc[KV];
#pragma unroll
    for (int k = 0; k < KV; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < ns; s0 += B) {
        float4 v[B][KV];
        float ls[B];
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const bool in = s0 + u < ns;
            ls[u] = in ? pl[s0 + u] : -INFINITY;
#pragma unroll
            for (int k = 0; k < KV; ++k)
                v[u][k] = in ? src[(int64_t)(s0 + u) * (DV / 4) + 32 * k]
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < B; ++u) {
            if (ls[u] == -INFINITY) continue;
            const float wgt = __expf(ls[u] - mx) * inv;
#pragma unroll
            for (int k = 0; k < KV; ++k) {
                acc[k].x += wgt * v[u][k].x;
                acc[k].y += wgt * v[u][k].y;
                acc[k].z += wgt * v[u][k].z;
                acc[k].w += wgt * v[u][k].w;
            }
        }
    }
    __nv_bfloat16 *o = a.out + rh * DV;
#pragma unroll
    for (int k = 0; k < KV; ++k) {
        const int d0 = 4 * (lane + 32 * (qd * KV + k));
        *reinterpret_cast<uint2 *>(o + d0) =
            make_uint2(pack_bf16(acc[k].x, acc[k].y), pack_bf16(acc[k].z, acc[k].w));
    }
    if (qd == 0 && lane == 0) a.lse[rh] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

cudaError_t launch_combine(const AttendArgs &a, int64_t rows, cudaStream_t s) {
    const int64_t n_rh = rows * a.H;
    if (a.n_split >= kCombineSplitMin) {
        const int64_t blocks = (n_rh * 4 + kCombineWarps - 1) / kCombineWarps;
        hfa_combine_kernel<true><<<(unsigned)blocks, 32 * kCombineWarps, 0, s>>>(a, n_rh);
    } else {
        const int64_t blocks = (n_rh + kCombineWarps - 1) / kCombineWarps;
        hfa_combine_kernel<false><<<(unsigned)blocks, 32 * kCombineWarps, 0, s>>>(a, n_rh);
    }
    return launched();
}

template <int NM>
size_t hfa_smem() {
    return (size_t)(16 * NM * SROW + STAGES * NK * SROW + 2 * NM * 16 * PROW) * 2 +
           (size_t)(2 * NM * 2 * 16) * 4 + (size_t)(STAGES * NK + 4) * 4;
}

template <int NM>
cudaError_t launch_nm(const AttendArgs &a, int64_t rows, cudaStream_t s) {
    const size_t smem = hfa_smem<NM>();
    cudaError_t e = cudaFuncSetAttribute(hfa_kernel<NM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int groups = (a.H + 16 * NM - 1) / (16 * NM);
    dim3 grid((unsigned)rows, (unsigned)groups, (unsigned)a.n_split);
    hfa_kernel<NM><<<grid, 64 * NM, smem, s>>>(a);
    return launched();
}

}  // namespace

int attend_heads_per_cta(int H) {
    const int nm = (H + 15) / 16;
    return 16 * (nm < 4 ? nm : 4);
}

cudaError_t launch_attend(const AttendArgs &a, int64_t rows, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    if (rows > 0x7FFFFFFF) return cudaErrorInvalidValue;
    cudaError_t e;
    if (a.use_tc) {
        e = launch_attend_tc(a, rows, s);
        if (e != cudaSuccess || a.n_split == 1) return e;
        return launch_combine(a, rows, s);
    }
    const int nm = attend_heads_per_cta(a.H) / 16;
    switch (nm) {
        case 1: e = launch_nm<1>(a, rows, s); break;
        case 2: e = launch_nm<2>(a, rows, s); break;
        case 3: e = launch_nm<3>(a, rows, s); break;
        default: e = launch_nm<4>(a, rows, s); break;
    }
    if (e != cudaSuccess || a.n_split == 1) return e;
    return launch_combine(a, rows, s);
}

}  // namespace lsa
