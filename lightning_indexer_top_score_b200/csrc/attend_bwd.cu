// attend_bwd.cu -- backward of the Hybrid Sparse Attention over absorbed-MLA latent rows.
//
// Paper: Sec. 2.2 (u_t = Attn over the latent rows c_s, s in S_t), Sec. 3.1 (S_t = sink U swa
// U S_sparse), Sec. 4.1.1 (HFA backward: gather for dQ, scatter-add of the row gradients; the
// window halves the scattered set), Table 2 (the training setting).  With z_s = scale q.c_s,
// p_s = exp(z_s - lse), dp_s = dout . c_s[0:Dv], D = sum_s p_s dp_s and dz_s = p_s (dp_s - D):
//   dq   = scale sum_s dz_s c_s
//   dc_s += scale dz_s q + p_s dout   (the second term on the first Dv dims)
//
// One CTA per (query row, group of 32 heads), 16 warps, over the row's virtual key list
// [sink | window | gathered] in tiles of 32 rows (the forward's order), double-buffered through
// cp.async.  The four contractions run on the tensor cores as warp-level m16n8k16 bf16 MMAs with
// fp32 accumulation:
//   S  = Q C^T    (32 heads x 32 keys, K = 576)   one 16x8 fragment per warp (warps 0-7)
//   dP = dO V^T   (32 x 32, K = 512)              one fragment per warp (warps 8-15)
//   dQ += dZ C    (32 x 576, K = 32 keys)         10 fragments per warp, held for the whole row
//   dC  = dZ^T Q + P^T dO  (32 keys x 576, K = 32 heads)  per 16-key half, then one 16-byte
//                                                  vector atomic per thread and fragment pair
// Given the forward's outputs, lse is taken as is and D = dout . out (the usual training path);
// otherwise a first pass over the keys recomputes each head's lse and D (online max / sums in
// fp32).  The main pass forms P and dZ = P (dP - D) scale, rounds both to bf16 (the operands of
// the dQ and dC products, as the forward rounds P for P V), and runs the two gradient products.
// Rows are padded so that the eight addresses of every ldmatrix phase fall in distinct bank
// groups.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int HG = 32;          // heads per CTA: two m16 tiles
constexpr int NK = 32;          // keys per tile
constexpr int QROW = DQK + 8;   // bf16 elements per padded q / key row: 1168 B
constexpr int OROW = DV + 8;    // 1040 B
constexpr int PROW = NK + 8;    // 80 B
constexpr int SROW = NK + 1;    // fp32 score rows
constexpr int kThreads = 512;
constexpr int kNt = DQK / 8;    // 72 column tiles of 8 dims
constexpr int kNtV = DV / 8;    // 64 of them inside the value dims
constexpr int kTilesPerWarp = 5;  // column tiles w + 16 i, i < 5 (i = 4 only for warps 0-7)
constexpr float kLog2e = 1.4426950408889634f;

struct Smem {
    __nv_bfloat16 q[HG][QROW];
    __nv_bfloat16 dout[HG][OROW];
    __nv_bfloat16 k[2][NK][QROW];
    float s[HG][SROW];
    float dp[HG][SROW];
    __nv_bfloat16 pb[HG][PROW];
    __nv_bfloat16 zb[HG][PROW];
    float lse2[HG];
    float D[HG];
    int32_t pos[2][NK];
};

__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

// d += a b for one m16n8k16 tile: a row-major 16x16, b column-major 16x8, bf16 in, fp32 out
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

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
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr(dst)), "l"(src),
                 "r"(bytes)
                 : "memory");
}

// Issues the copies of tile `tile` into stage st (all threads) and records its positions;
// absent keys (past the row's list) are zero-filled and get position -1.
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

// S (warps 0-7) or dP (warps 8-15): one 16 heads x 8 keys fragment per warp, written to shared
// memory in fp32.  Two accumulators (even / odd k-steps) halve the dependent MMA chain, and the
// fragments of the next pair of k-steps are loaded while the current pair multiplies.
__device__ __forceinline__ void scores_phase(Smem &S, int st, int warp, int lane) {
    const bool is_s = warp < 8;
    const int f = warp & 7, m = f >> 2, n = f & 3;
    const int ksteps = is_s ? DQK / 16 : DV / 16;  // 36 or 32: multiples of 4
    const uint32_t a0 = is_s ? saddr(&S.q[m * 16 + (lane & 15)][(lane >> 4) * 8])
                             : saddr(&S.dout[m * 16 + (lane & 15)][(lane >> 4) * 8]);
    // one x4 load covers the B fragments of two k-steps: lanes 8q..8q+7 address key rows
    // n*8 + 0..7 at dims 8q (+ 32 per pair of k-steps)
    const uint32_t b0 = saddr(&S.k[st][n * 8 + (lane & 7)][(lane >> 3) * 8]);
    float e[4] = {0.f, 0.f, 0.f, 0.f}, o[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t fa[2][4], fa2[2][4], fb[2][4];
    ldsm_x4(fb[0], b0);
    ldsm_x4(fa[0], a0);
    ldsm_x4(fa2[0], a0 + 32);
    for (int kk = 0; kk < ksteps; kk += 4) {
        ldsm_x4(fb[1], b0 + (kk + 2) * 32);
        ldsm_x4(fa[1], a0 + (kk + 2) * 32);
        ldsm_x4(fa2[1], a0 + (kk + 3) * 32);
        mma_bf16(e, fa[0], fb[0][0], fb[0][1]);
        mma_bf16(o, fa2[0], fb[0][2], fb[0][3]);
        if (kk + 4 < ksteps) {
            ldsm_x4(fb[0], b0 + (kk + 4) * 32);
            ldsm_x4(fa[0], a0 + (kk + 4) * 32);
            ldsm_x4(fa2[0], a0 + (kk + 5) * 32);
        }
        mma_bf16(e, fa[1], fb[1][0], fb[1][1]);
        mma_bf16(o, fa2[1], fb[1][2], fb[1][3]);
    }
    float(*out)[SROW] = is_s ? S.s : S.dp;
    const int row = m * 16 + (lane >> 2), col = n * 8 + 2 * (lane & 3);
    out[row][col] = e[0] + o[0];
    out[row][col + 1] = e[1] + o[1];
    out[row + 8][col] = e[2] + o[2];
    out[row + 8][col + 1] = e[3] + o[3];
}

// Pass 1 (no forward outputs given): each head's lse and D = sum_s p_s dp_s by an online max /
// sum over the tiles, 16 threads per head (uniform after each tile), into S.lse2 / S.D.
__device__ __forceinline__ void pass1_stats(Smem &S, const BwdArgs &a, int64_t r, int64_t b,
                                            const Regions &g, int64_t n_sp, int64_t n_tiles,
                                            float sl2, int warp, int lane, int eh, int ej) {
    const int tid = threadIdx.x;
    float m = -INFINITY, l = 0.f, gsum = 0.f;
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
        scores_phase(S, st, warp, lane);
        __syncthreads();
        const bool v0 = S.pos[st][ej] >= 0, v1 = S.pos[st][ej + 1] >= 0;
        const float z0 = v0 ? S.s[eh][ej] * sl2 : -INFINITY;  // log2 units
        const float z1 = v1 ? S.s[eh][ej + 1] * sl2 : -INFINITY;
        float mt = fmaxf(z0, z1);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, o));
        const float mn = fmaxf(m, mt);
        const float e0 = (v0 && mn > -INFINITY) ? exp2f(z0 - mn) : 0.f;
        const float e1 = (v1 && mn > -INFINITY) ? exp2f(z1 - mn) : 0.f;
        float es = e0 + e1, ed = e0 * S.dp[eh][ej] + e1 * S.dp[eh][ej + 1];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
            es += __shfl_xor_sync(0xFFFFFFFFu, es, o);
            ed += __shfl_xor_sync(0xFFFFFFFFu, ed, o);
        }
        const float alpha = (m > -INFINITY) ? exp2f(m - mn) : 0.f;
        l = l * alpha + es;
        gsum = gsum * alpha + ed;
        m = mn;
        __syncthreads();  // scores, positions and the stage are rewritten by the next tile
    }
    if ((tid & 15) == 0) {
        S.lse2[eh] = (l > 0.f) ? m + log2f(l) : INFINITY;  // exp2(z - lse2) = p; no keys: p = 0
        S.D[eh] = (l > 0.f) ? gsum / l : 0.f;
        if (!isfinite(l) || !isfinite(gsum)) raise_error(a.err, LSA_DEVERR_NONFINITE);
    }
}

__global__ void __launch_bounds__(kThreads, 1) hfa_bwd_kernel(BwdArgs a) {
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
    // this row's q and dout for the 32 heads of the group, into padded rows
    {
        const uint4 *qg = reinterpret_cast<const uint4 *>(a.q + (r * a.H + h0) * (int64_t)DQK);
        for (int e = tid; e < HG * DQK / 8; e += kThreads) {
            const int h = e / (DQK / 8), c8 = e - h * (DQK / 8);
            *reinterpret_cast<uint4 *>(&S.q[h][c8 * 8]) = qg[e];
        }
        const uint4 *dg = reinterpret_cast<const uint4 *>(a.dout + (r * a.H + h0) * (int64_t)DV);
        for (int e = tid; e < HG * DV / 8; e += kThreads) {
            const int h = e / (DV / 8), c8 = e - h * (DV / 8);
            *reinterpret_cast<uint4 *>(&S.dout[h][c8 * 8]) = dg[e];
        }
    }
    __syncthreads();
    const int64_t n_sp = nsp_s;
    const int64_t n_total = g.sink_hi + (g.swa_hi - g.swa_lo) + n_sp;
    const int64_t n_tiles = (n_total + NK - 1) / NK;
    const float sl2 = a.scale * kLog2e;
    // element phases: thread (head eh, keys ej, ej + 1)
    const int eh = tid >> 4, ej = (tid & 15) * 2;

    if (a.lse != nullptr) {
        // the forward's lse, and D = dout . out over the value dims (two heads per warp)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int hh = warp * 2 + u;
            const uint4 *orow = reinterpret_cast<const uint4 *>(
                a.o + (r * a.H + h0 + hh) * (int64_t)DV + lane * 16);
            const uint4 *drow = reinterpret_cast<const uint4 *>(&S.dout[hh][lane * 16]);
            float acc = 0.f;
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                const uint4 ov = orow[v], dv = drow[v];
                const __nv_bfloat162 *o2 = reinterpret_cast<const __nv_bfloat162 *>(&ov);
                const __nv_bfloat162 *d2 = reinterpret_cast<const __nv_bfloat162 *>(&dv);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 of = __bfloat1622float2(o2[k]), df = __bfloat1622float2(d2[k]);
                    acc = fmaf(of.x, df.x, fmaf(of.y, df.y, acc));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
            if (lane == 0) {
                const float ls = a.lse[r * a.H + h0 + hh];
                S.lse2[hh] = (ls > -INFINITY) ? ls * kLog2e : INFINITY;  // no keys: p = 0
                S.D[hh] = acc;
                if (!isfinite(acc) || ls != ls || ls == INFINITY)
                    raise_error(a.err, LSA_DEVERR_NONFINITE);
            }
        }
    } else {
        pass1_stats(S, a, r, b, g, n_sp, n_tiles, sl2, warp, lane, eh, ej);
    }
    __syncthreads();
    const float lse2 = S.lse2[eh], Dh = S.D[eh];

    // ---------------- pass 2: dq and the row gradients
    const int gq = lane >> 2, cq = lane & 3;
    const int n_mine = warp < kNt - 4 * 16 ? kTilesPerWarp : kTilesPerWarp - 1;
    float dq[kTilesPerWarp][2][4];
#pragma unroll
    for (int i = 0; i < kTilesPerWarp; ++i)
#pragma unroll
        for (int mm = 0; mm < 2; ++mm)
#pragma unroll
            for (int k = 0; k < 4; ++k) dq[i][mm][k] = 0.f;
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
        scores_phase(S, st, warp, lane);
        __syncthreads();
        {
            const bool v0 = S.pos[st][ej] >= 0, v1 = S.pos[st][ej + 1] >= 0;
            const float p0 = v0 ? exp2f(S.s[eh][ej] * sl2 - lse2) : 0.f;
            const float p1 = v1 ? exp2f(S.s[eh][ej + 1] * sl2 - lse2) : 0.f;
            const float z0 = p0 * (S.dp[eh][ej] - Dh) * a.scale;
            const float z1 = p1 * (S.dp[eh][ej + 1] - Dh) * a.scale;
            *reinterpret_cast<__nv_bfloat162 *>(&S.pb[eh][ej]) = __floats2bfloat162_rn(p0, p1);
            *reinterpret_cast<__nv_bfloat162 *>(&S.zb[eh][ej]) = __floats2bfloat162_rn(z0, z1);
        }
        __syncthreads();
        // dq[heads, dims] += dZ[heads, keys] C[keys, dims]
        {
            uint32_t az[2][2][4];  // [head half][key half]
#pragma unroll
            for (int mm = 0; mm < 2; ++mm)
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    ldsm_x4(az[mm][kk],
                            saddr(&S.zb[mm * 16 + (lane & 15)][kk * 16 + (lane >> 4) * 8]));
#pragma unroll
            for (int i = 0; i < kTilesPerWarp; ++i) {
                if (i < n_mine) {
                    const int nt = warp + 16 * i;
                    uint32_t fb[4];  // key rows 0-7, 8-15, 16-23, 24-31 at dims nt*8
                    ldsm_x4_t(fb, saddr(&S.k[st][lane][nt * 8]));
#pragma unroll
                    for (int mm = 0; mm < 2; ++mm) {
                        mma_bf16(dq[i][mm], az[mm][0], fb[0], fb[1]);
                        mma_bf16(dq[i][mm], az[mm][1], fb[2], fb[3]);
                    }
                }
            }
        }
        // dC[keys, dims] = dZ^T[keys, heads] Q[heads, dims] + P^T dO, one 16-key half at a time:
        // every product of the half first, then the scatter (an atomic between two fragment
        // loads would hold the next load until the product feeding it is done)
#pragma unroll
        for (int mk = 0; mk < 2; ++mk) {
            uint32_t az[2][4], ap[2][4];  // [head half]
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) {
                const int hr = kh * 16 + ((lane >> 4) << 3) + (lane & 7);
                const int kc = mk * 16 + ((lane >> 3) & 1) * 8;
                ldsm_x4_t(az[kh], saddr(&S.zb[hr][kc]));
                ldsm_x4_t(ap[kh], saddr(&S.pb[hr][kc]));
            }
            float acc[kTilesPerWarp][4];
#pragma unroll
            for (int i = 0; i < kTilesPerWarp; ++i) {
                acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
                if (i < n_mine) {
                    const int nt = warp + 16 * i;
                    uint32_t fq[4];  // head rows 0-7 .. 24-31 at dims nt*8
                    ldsm_x4_t(fq, saddr(&S.q[lane][nt * 8]));
                    mma_bf16(acc[i], az[0], fq[0], fq[1]);
                    mma_bf16(acc[i], az[1], fq[2], fq[3]);
                    if (nt < kNtV) {
                        uint32_t fo[4];
                        ldsm_x4_t(fo, saddr(&S.dout[lane][nt * 8]));
                        mma_bf16(acc[i], ap[0], fo[0], fo[1]);
                        mma_bf16(acc[i], ap[1], fo[2], fo[3]);
                    }
                }
            }
            // lane pairs (c, c^1) swap halves so that each lane holds four consecutive dims of
            // one key: even lanes row g, odd lanes row g + 8
            const bool even = !(cq & 1);
            const int key = mk * 16 + gq + (even ? 0 : 8);
            const int64_t pos = S.pos[st][key];
            float *row = dc_seq + (pos >= 0 ? pos : 0) * DQK + 2 * (cq & ~1);
#pragma unroll
            for (int i = 0; i < kTilesPerWarp; ++i) {
                if (i < n_mine) {
                    const float s0 = even ? acc[i][2] : acc[i][0];
                    const float s1 = even ? acc[i][3] : acc[i][1];
                    const float r0 = __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
                    const float r1 = __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
                    if (pos >= 0) {
                        const float4 v = even ? make_float4(acc[i][0], acc[i][1], r0, r1)
                                              : make_float4(r0, r1, acc[i][2], acc[i][3]);
                        atomicAdd(reinterpret_cast<float4 *>(row + (warp + 16 * i) * 8), v);
                    }
                }
            }
        }
        __syncthreads();  // p / dz, scores and the stage are reused by the next tile
    }
#pragma unroll
    for (int i = 0; i < kTilesPerWarp; ++i) {
        if (i < n_mine) {
            const int col = (warp + 16 * i) * 8 + 2 * cq;
#pragma unroll
            for (int mm = 0; mm < 2; ++mm) {
                float *d0 = a.dq + (r * a.H + h0 + mm * 16 + gq) * (int64_t)DQK + col;
                *reinterpret_cast<float2 *>(d0) = make_float2(dq[i][mm][0], dq[i][mm][1]);
                *reinterpret_cast<float2 *>(d0 + 8 * DQK) =
                    make_float2(dq[i][mm][2], dq[i][mm][3]);
            }
        }
    }
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
