// attend_bwd.cu -- backward of the Hybrid Sparse Attention over absorbed-MLA latent rows.
//
// Paper: Sec. 2.2 (u_t = Attn over the latent rows c_s, s in S_t), Sec. 3.1 (S_t = sink U swa
// U S_sparse), Sec. 4.1.1 (HFA backward: gather for dQ, scatter-add of the row gradients; the
// window halves the scattered set), Table 2 (the training setting).  With z_s = scale q.c_s,
// p_s = exp(z_s - lse), dp_s = dout . c_s[0:Dv], D = sum_s p_s dp_s and dz_s = p_s (dp_s - D):
//   dq   = scale sum_s dz_s c_s
//   dc_s += scale dz_s q + p_s dout   (the second term on the first Dv dims)
//
// One CTA per (query row, group of 32 heads) walks the row's virtual key list [sink | window |
// gathered] in tiles of 32 rows (the forward's order).  The contractions run on the tensor cores
// as warp-level m16n8k16 bf16 MMAs with fp32 accumulation, in a warp-specialised pipeline:
//   score warps 0-3     S = Q C^T (K = 576) or dP = dO V^T (K = 512) for 16 heads x 32 keys
//                       each (four fragments sharing every A fragment), then P (S warps) and
//                       dZ = P (dP - D) scale (dP warps) in registers, rounded to bf16 into a
//                       double-buffered tile of P / dZ;
//   gradient warps 4-15 the gathers (cp.async, two tiles ahead, three stages), then for the tile
//                       the score warps finished: dQ += dZ C (dq fragments held in registers for
//                       the whole row) and dC = dZ^T Q + P^T dO per 16-key half, staged per warp
//                       in shared memory and scattered with 16-byte vector atomics, row by row.
// The roles hand tiles over through mbarriers (full: the gather landed; pready: P / dZ written;
// pfree: the gradient warps are done with a P / dZ buffer).  Every wait is bounded; a role that
// gives up votes with the rest of its role (bar.red.and) so that all of it leaves together.
// Given the forward's outputs, lse is taken as is and D = dout . out (the usual training path);
// otherwise a first pass over the keys with all 16 warps recomputes each head's lse and D
// (online max / sums in fp32).  P and dZ are rounded to bf16 as the operands of the gradient
// products, as the forward rounds P for P V.  Rows are padded so that the eight addresses of
// every ldmatrix phase fall in distinct bank groups.
#include "lsa_internal.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using tc::cp_async_arrive_noinc;
using tc::cp_async_wait_all;
using tc::mbar_arrive;
using tc::mbar_init;
using tc::mbar_wait;

constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int HG = 32;          // heads per CTA: two m16 tiles
constexpr int NK = 32;          // keys per tile
constexpr int QROW = DQK + 8;   // bf16 elements per padded q / key row: 1168 B
constexpr int OROW = DV + 8;    // 1040 B
constexpr int PROW = NK + 8;    // 80 B
constexpr int SROW = NK + 8;    // fp32 rows of the score / p tiles (float2-aligned)
constexpr int STAGES = 3;       // key-tile ring of the main pass
constexpr int kThreads = 512;
constexpr int kScoreWarps = 4;
constexpr int kGradThreads = kThreads - 32 * kScoreWarps;  // 384
constexpr int kGradWarps = kGradThreads / 32;              // 12
constexpr int kNt = DQK / 8;    // 72 column tiles of 8 dims
constexpr int kNtV = DV / 8;    // 64 of them inside the value dims
constexpr int kTilesPerWarp = kNt / kGradWarps;  // 6: dq tiles gw + 12 j; dC tiles 6 gw + j
constexpr int kStageRow = 52;    // a warp's 48 dC dims, padded to 16-byte aligned rows
constexpr int kIdxCache = 2048;  // index rows up to this long are read from shared memory
constexpr float kLog2e = 1.4426950408889634f;
// named barriers (0 is __syncthreads)
constexpr int kBarGrad = 1, kBarScore = 2, kBarPair = 3;  // pairs: 3 + head half

struct Smem {
    __nv_bfloat16 q[HG][QROW];
    __nv_bfloat16 dout[HG][OROW];
    __nv_bfloat16 k[STAGES][NK][QROW];
    float sc[2][HG][SROW];  // first pass: scores / dP; main pass: p of P / dZ buffers 0 and 1
    __nv_bfloat16 pb[2][HG][PROW];
    __nv_bfloat16 zb[2][HG][PROW];
    float stage[kGradWarps][8][kStageRow];  // per gradient warp: 8 keys x 48 dC dims
    int32_t idx_s[kIdxCache];  // the row's gathered positions (when K <= kIdxCache)
    float lse2[HG];
    float D[HG];
    int32_t pos[STAGES][NK];
    uint64_t full[STAGES];
    uint64_t pready[2];
    uint64_t pfree[2];
    int abort;
    int nsp;
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

__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Named barrier over n threads that also ANDs a predicate across them: every participant gets
// the same answer, so a role can leave its loop as one.
__device__ __forceinline__ bool named_and(int id, int n, bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void cp16(void *dst, const void *src, int bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr(dst)), "l"(src),
                 "r"(bytes)
                 : "memory");
}

// Copies of one tile's key rows into stage st by threads [0, nthr) of a group (thread index
// gt); absent keys (past the row's list) are zero-filled.  Positions must be in S.pos[st].
__device__ __forceinline__ void copy_tile(Smem &S, int st, const __nv_bfloat16 *cseq, int gt,
                                          int nthr) {
    for (int e = gt; e < NK * (DQK / 8); e += nthr) {
        const int j = e / (DQK / 8), pc = e - j * (DQK / 8);
        const int64_t pos = S.pos[st][j];
        cp16(&S.k[st][j][pc * 8], pos >= 0 ? cseq + pos * DQK + pc * 8 : cseq, pos >= 0 ? 16 : 0);
    }
}

// ---------------------------------------------------------------- first pass (no forward outputs)

// All threads: tile `tile` into stage st (of the first two), positions first.
__device__ __forceinline__ void load_tile_all(Smem &S, int st, const BwdArgs &a,
                                              const int32_t *idx, const __nv_bfloat16 *cseq,
                                              const Regions &g, int64_t n_sp, int64_t tile) {
    const int tid = threadIdx.x;
    if (tid < NK) S.pos[st][tid] = (int32_t)bwd_key_pos(a.err, idx, g, n_sp, tile * NK + tid);
    __syncthreads();  // positions visible to every copying thread
    copy_tile(S, st, cseq, tid, kThreads);
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// S (warps 0-7) or dP (warps 8-15): one 16 heads x 8 keys fragment per warp into S.sc[0] /
// S.sc[1] in fp32 (the first pass only needs the scores, not the gradient operands).  The
// k-steps accumulate in one chain in order, as in the main pass, so both passes get the same
// bits (a single-key row then has D = dp exactly and dz = 0).
__device__ __forceinline__ void scores_all(Smem &S, int st, int warp, int lane) {
    const bool is_s = warp < 8;
    const int f = warp & 7, m = f >> 2, n = f & 3;
    const int ksteps = is_s ? DQK / 16 : DV / 16;
    const uint32_t a0 = is_s ? saddr(&S.q[m * 16 + (lane & 15)][(lane >> 4) * 8])
                             : saddr(&S.dout[m * 16 + (lane & 15)][(lane >> 4) * 8]);
    const uint32_t b0 = saddr(&S.k[st][n * 8 + (lane & 7)][(lane >> 3) * 8]);
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    for (int kk = 0; kk < ksteps; kk += 2) {
        uint32_t fa[4], fa2[4], fb[4];
        ldsm_x4(fb, b0 + kk * 32);
        ldsm_x4(fa, a0 + kk * 32);
        ldsm_x4(fa2, a0 + (kk + 1) * 32);
        mma_bf16(e, fa, fb[0], fb[1]);
        mma_bf16(e, fa2, fb[2], fb[3]);
    }
    float(*out)[SROW] = S.sc[is_s ? 0 : 1];
    const int row = m * 16 + (lane >> 2), col = n * 8 + 2 * (lane & 3);
    *reinterpret_cast<float2 *>(&out[row][col]) = make_float2(e[0], e[1]);
    *reinterpret_cast<float2 *>(&out[row + 8][col]) = make_float2(e[2], e[3]);
}

// Each head's lse (log2 units) and D = sum_s p_s dp_s by an online max / sum over the tiles,
// 16 threads per head (uniform after each tile), into S.lse2 / S.D.
__device__ __forceinline__ void first_pass(Smem &S, const BwdArgs &a, const int32_t *idx,
                                           const __nv_bfloat16 *cseq, const Regions &g,
                                           int64_t n_sp, int64_t n_tiles, float sl2) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int eh = tid >> 4, ej = (tid & 15) * 2;
    float m = -INFINITY, l = 0.f, gsum = 0.f;
    if (n_tiles > 0) load_tile_all(S, 0, a, idx, cseq, g, n_sp, 0);
    for (int64_t it = 0; it < n_tiles; ++it) {
        const int st = (int)(it & 1);
        if (it + 1 < n_tiles) {
            load_tile_all(S, st ^ 1, a, idx, cseq, g, n_sp, it + 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        scores_all(S, st, warp, lane);
        __syncthreads();
        const bool v0 = S.pos[st][ej] >= 0, v1 = S.pos[st][ej + 1] >= 0;
        const float z0 = v0 ? S.sc[0][eh][ej] * sl2 : -INFINITY;  // log2 units
        const float z1 = v1 ? S.sc[0][eh][ej + 1] * sl2 : -INFINITY;
        float mt = fmaxf(z0, z1);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, o));
        const float mn = fmaxf(m, mt);
        const float e0 = (v0 && mn > -INFINITY) ? exp2f(z0 - mn) : 0.f;
        const float e1 = (v1 && mn > -INFINITY) ? exp2f(z1 - mn) : 0.f;
        float es = e0 + e1, ed = e0 * S.sc[1][eh][ej] + e1 * S.sc[1][eh][ej + 1];
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

// ---------------------------------------------------------------- main pass, gradient warps

// Issues tile `tile` into stage st: positions (first warp of the role), then the copies of all
// gradient threads, each of which arrives on full[st] once its own copies have landed.  The
// stage's previous tile is still read by the other gradient warps (its positions address their
// row-gradient scatter) until they reach the first barrier, so nothing of the stage, positions
// included, is written before it.
__device__ __forceinline__ void issue_tile(Smem &S, int st, const BwdArgs &a, const int32_t *idx,
                                           const __nv_bfloat16 *cseq, const Regions &g,
                                           int64_t n_sp, int64_t tile, int gt) {
    named_sync(kBarGrad, kGradThreads);  // every gradient warp is done with the stage
    if (gt < NK) {
        S.pos[st][gt] = (int32_t)bwd_key_pos(a.err, idx, g, n_sp, tile * NK + gt);
        mbar_arrive(&S.full[st]);  // releases the position
    }
    named_sync(kBarGrad, kGradThreads);  // positions visible to every copying thread
    copy_tile(S, st, cseq, gt, kGradThreads);
    cp_async_arrive_noinc(&S.full[st]);
}

// ---------------------------------------------------------------- kernel

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
        // the row has no keys: its dq slice is written as zeros, no latent row is touched
        float *dq = a.dq + (r * a.H + h0) * (int64_t)DQK;
        for (int i = tid; i < HG * DQK; i += kThreads) dq[i] = 0.f;
        return;
    }
    const Regions g = regions_of(t, a.Ks, a.Kw);
    const __nv_bfloat16 *cseq = a.c + b * a.L_max * DQK;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(&S.full[s], kGradThreads + NK);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&S.pready[s], 32 * kScoreWarps);
            mbar_init(&S.pfree[s], kGradThreads);
        }
        S.abort = 0;
        S.nsp = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // gathered picks of this row: the selection writes them ascending, -1 after the last.
    // A row of up to kIdxCache entries is kept in shared memory for the tile positions.
    const bool idx_cached = a.K <= kIdxCache;
    {
        int c = 0;
        for (int i = tid; i < a.K; i += kThreads) {
            const int32_t v = a.idx[r * a.K + i];
            if (idx_cached) S.idx_s[i] = v;
            c += (v >= 0);
        }
        if (c) atomicAdd(&S.nsp, c);
    }
    const int32_t *idx = idx_cached ? S.idx_s : a.idx + r * a.K;
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
    const int64_t n_sp = S.nsp;
    const int64_t n_tiles = (g.sink_hi + (g.swa_hi - g.swa_lo) + n_sp + NK - 1) / NK;
    const float sl2 = a.scale * kLog2e;

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
        first_pass(S, a, idx, cseq, g, n_sp, n_tiles, sl2);
    }
    __syncthreads();
    const int gq = lane >> 2, cq = lane & 3;

    if (warp < kScoreWarps) {
        // ================= score warps: warp (mat, m) -> S (mat 0) or dP (mat 1), heads m*16..
        const int mat = warp >> 1, m = warp & 1;
        const int ksteps = mat ? DV / 16 : DQK / 16;  // 32 or 36 k-steps
        const uint32_t a0 = mat ? saddr(&S.dout[m * 16 + (lane & 15)][(lane >> 4) * 8])
                                : saddr(&S.q[m * 16 + (lane & 15)][(lane >> 4) * 8]);
        // B: key rows kb + (lane>>4)*8 + (lane&7) at dims ((lane>>3)&1)*8: one x4 load holds
        // two 8-key fragments (keys kb..kb+7, kb+8..kb+15) for one k-step
        const int brow = ((lane >> 4) << 3) + (lane & 7), bcol = ((lane >> 3) & 1) * 8;
        const int hr0 = m * 16 + gq;  // the thread's heads: hr0 and hr0 + 8
        const float lse_a = S.lse2[hr0], lse_b = S.lse2[hr0 + 8];
        const float D_a = S.D[hr0], D_b = S.D[hr0 + 8];
        for (int64_t it = 0; it < n_tiles; ++it) {
            const int st = (int)(it % STAGES), buf = (int)(it & 1);
            bool ok = mbar_wait(&S.full[st], (uint32_t)((it / STAGES) & 1), &S.abort, a.err);
            if (it >= 2)
                ok = ok && mbar_wait(&S.pfree[buf], (uint32_t)(((it - 2) >> 1) & 1), &S.abort,
                                     a.err);
            if (!named_and(kBarScore, 32 * kScoreWarps, ok)) break;
            float acc[4][4];
#pragma unroll
            for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
            const uint32_t b0 = saddr(&S.k[st][brow][bcol]);
            const uint32_t b1 = saddr(&S.k[st][16 + brow][bcol]);
            uint32_t fa[2][4], fb[2][2][4];
            ldsm_x4(fa[0], a0);
            ldsm_x4(fb[0][0], b0);
            ldsm_x4(fb[0][1], b1);
            for (int kk = 0; kk < ksteps; kk += 2) {
                // k-step kk from buffer 0 while kk + 1 loads into buffer 1, then the reverse
                ldsm_x4(fa[1], a0 + (kk + 1) * 32);
                ldsm_x4(fb[1][0], b0 + (kk + 1) * 32);
                ldsm_x4(fb[1][1], b1 + (kk + 1) * 32);
                mma_bf16(acc[0], fa[0], fb[0][0][0], fb[0][0][1]);
                mma_bf16(acc[1], fa[0], fb[0][0][2], fb[0][0][3]);
                mma_bf16(acc[2], fa[0], fb[0][1][0], fb[0][1][1]);
                mma_bf16(acc[3], fa[0], fb[0][1][2], fb[0][1][3]);
                if (kk + 2 < ksteps) {
                    ldsm_x4(fa[0], a0 + (kk + 2) * 32);
                    ldsm_x4(fb[0][0], b0 + (kk + 2) * 32);
                    ldsm_x4(fb[0][1], b1 + (kk + 2) * 32);
                }
                mma_bf16(acc[0], fa[1], fb[1][0][0], fb[1][0][1]);
                mma_bf16(acc[1], fa[1], fb[1][0][2], fb[1][0][3]);
                mma_bf16(acc[2], fa[1], fb[1][1][0], fb[1][1][1]);
                mma_bf16(acc[3], fa[1], fb[1][1][2], fb[1][1][3]);
            }
            // fragment n holds keys n*8 + 2 cq, +1 of heads hr0 (acc 0, 1) and hr0 + 8 (acc 2, 3)
            if (mat == 0) {
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const int key = n * 8 + 2 * cq;
                    const bool v0 = S.pos[st][key] >= 0, v1 = S.pos[st][key + 1] >= 0;
                    const float p0 = v0 ? exp2f(acc[n][0] * sl2 - lse_a) : 0.f;
                    const float p1 = v1 ? exp2f(acc[n][1] * sl2 - lse_a) : 0.f;
                    const float p2 = v0 ? exp2f(acc[n][2] * sl2 - lse_b) : 0.f;
                    const float p3 = v1 ? exp2f(acc[n][3] * sl2 - lse_b) : 0.f;
                    *reinterpret_cast<float2 *>(&S.sc[buf][hr0][key]) = make_float2(p0, p1);
                    *reinterpret_cast<float2 *>(&S.sc[buf][hr0 + 8][key]) = make_float2(p2, p3);
                    *reinterpret_cast<__nv_bfloat162 *>(&S.pb[buf][hr0][key]) =
                        __floats2bfloat162_rn(p0, p1);
                    *reinterpret_cast<__nv_bfloat162 *>(&S.pb[buf][hr0 + 8][key]) =
                        __floats2bfloat162_rn(p2, p3);
                }
                named_sync(kBarPair + m, 64);  // p of these heads ready for the dP warp
            } else {
                named_sync(kBarPair + m, 64);
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const int key = n * 8 + 2 * cq;
                    const float2 pa = *reinterpret_cast<const float2 *>(&S.sc[buf][hr0][key]);
                    const float2 pc = *reinterpret_cast<const float2 *>(&S.sc[buf][hr0 + 8][key]);
                    *reinterpret_cast<__nv_bfloat162 *>(&S.zb[buf][hr0][key]) =
                        __floats2bfloat162_rn(pa.x * (acc[n][0] - D_a) * a.scale,
                                              pa.y * (acc[n][1] - D_a) * a.scale);
                    *reinterpret_cast<__nv_bfloat162 *>(&S.zb[buf][hr0 + 8][key]) =
                        __floats2bfloat162_rn(pc.x * (acc[n][2] - D_b) * a.scale,
                                              pc.y * (acc[n][3] - D_b) * a.scale);
                }
            }
            mbar_arrive(&S.pready[buf]);
        }
        return;
    }

    // ================= gradient warps
    const int gt = tid - 32 * kScoreWarps, gw = gt >> 5;
    float dq[kTilesPerWarp][2][4];
#pragma unroll
    for (int j = 0; j < kTilesPerWarp; ++j)
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) dq[j][mm][0] = dq[j][mm][1] = dq[j][mm][2] = dq[j][mm][3] = 0.f;
    float *dc_seq = a.dc + b * a.L_max * DQK;
    for (int64_t i = 0; i < 2 && i < n_tiles; ++i)
        issue_tile(S, (int)i, a, idx, cseq, g, n_sp, i, gt);
    bool ok = true;
    for (int64_t it = 0; it < n_tiles; ++it) {
        const int st = (int)(it % STAGES), buf = (int)(it & 1);
        if (it + 2 < n_tiles)
            issue_tile(S, (int)((it + 2) % STAGES), a, idx, cseq, g, n_sp, it + 2, gt);
        ok = mbar_wait(&S.full[st], (uint32_t)((it / STAGES) & 1), &S.abort, a.err) &&
             mbar_wait(&S.pready[buf], (uint32_t)((it >> 1) & 1), &S.abort, a.err);
        if (!named_and(kBarGrad, kGradThreads, ok)) {
            ok = false;
            break;
        }
        // dq[heads, dims] += dZ[heads, keys] C[keys, dims]
        {
            uint32_t az[2][2][4];  // [head half][key half]
#pragma unroll
            for (int mm = 0; mm < 2; ++mm)
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    ldsm_x4(az[mm][kk],
                            saddr(&S.zb[buf][mm * 16 + (lane & 15)][kk * 16 + (lane >> 4) * 8]));
            // B fragments (key rows 0-7, 8-15, 16-23, 24-31 at dims nt*8) one column tile ahead
            const uint32_t kb = saddr(&S.k[st][lane][gw * 8]);
            uint32_t fb[2][4];
            ldsm_x4_t(fb[0], kb);
#pragma unroll
            for (int j = 0; j < kTilesPerWarp; ++j) {
                if (j + 1 < kTilesPerWarp) ldsm_x4_t(fb[(j + 1) & 1], kb + (j + 1) * kGradWarps * 16);
#pragma unroll
                for (int mm = 0; mm < 2; ++mm) {
                    mma_bf16(dq[j][mm], az[mm][0], fb[j & 1][0], fb[j & 1][1]);
                    mma_bf16(dq[j][mm], az[mm][1], fb[j & 1][2], fb[j & 1][3]);
                }
            }
        }
        // dC[keys, dims] = dZ^T[keys, heads] Q[heads, dims] + P^T dO.  Warp gw owns the 48
        // contiguous dims of tiles 6 gw .. 6 gw + 5.  Each block of 8 keys x 48 dims is staged
        // in the warp's shared tile and scattered row by row: a 16-byte vector atomic per lane,
        // the lanes of one instruction on about three rows of 192 contiguous bytes (a
        // fragment's own layout would put them on 16 rows of 32 bytes)
        float(*stg)[kStageRow] = S.stage[gw];
        float *col0 = dc_seq + 48 * gw;
#pragma unroll
        for (int mk = 0; mk < 2; ++mk) {
            uint32_t az[2][4], ap[2][4];  // [head half]
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) {
                const int hr = kh * 16 + ((lane >> 4) << 3) + (lane & 7);
                const int kc = mk * 16 + ((lane >> 3) & 1) * 8;
                ldsm_x4_t(az[kh], saddr(&S.zb[buf][hr][kc]));
                ldsm_x4_t(ap[kh], saddr(&S.pb[buf][hr][kc]));
            }
            // B fragments (head rows 0-7 .. 24-31 at dims nt*8) one column tile ahead
            const int nt0 = 6 * gw;
            const uint32_t qb = saddr(&S.q[lane][nt0 * 8]), ob = saddr(&S.dout[lane][nt0 * 8]);
            float acc[kTilesPerWarp][4];
            uint32_t fq[2][4], fo[2][4];
            ldsm_x4_t(fq[0], qb);
            if (nt0 < kNtV) ldsm_x4_t(fo[0], ob);
#pragma unroll
            for (int j = 0; j < kTilesPerWarp; ++j) {
                const int nt = nt0 + j;
                if (j + 1 < kTilesPerWarp) {
                    ldsm_x4_t(fq[(j + 1) & 1], qb + (j + 1) * 16);
                    if (nt + 1 < kNtV) ldsm_x4_t(fo[(j + 1) & 1], ob + (j + 1) * 16);
                }
                acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
                mma_bf16(acc[j], az[0], fq[j & 1][0], fq[j & 1][1]);
                mma_bf16(acc[j], az[1], fq[j & 1][2], fq[j & 1][3]);
                if (nt < kNtV) {
                    mma_bf16(acc[j], ap[0], fo[j & 1][0], fo[j & 1][1]);
                    mma_bf16(acc[j], ap[1], fo[j & 1][2], fo[j & 1][3]);
                }
            }
#pragma unroll
            for (int rh = 0; rh < 2; ++rh) {  // keys mk*16 + rh*8 + 0..7
#pragma unroll
                for (int j = 0; j < kTilesPerWarp; ++j)
                    *reinterpret_cast<float2 *>(&stg[gq][j * 8 + 2 * cq]) =
                        make_float2(acc[j][2 * rh], acc[j][2 * rh + 1]);
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const int f = k * 32 + lane, rr = f / 12, q4 = f - rr * 12;
                    const float4 v = *reinterpret_cast<const float4 *>(&stg[rr][q4 * 4]);
                    const int64_t pos = S.pos[st][mk * 16 + rh * 8 + rr];
                    if (pos >= 0)
                        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(
                                         col0 + pos * DQK + q4 * 4),
                                     "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                                     : "memory");
                }
                __syncwarp();  // the tile is rewritten by the next block
            }
        }
        mbar_arrive(&S.pfree[buf]);
    }
    cp_async_wait_all();  // none of this thread's copies may still be in flight at exit
    if (!ok) return;
#pragma unroll
    for (int j = 0; j < kTilesPerWarp; ++j) {
        const int col = (gw + kGradWarps * j) * 8 + 2 * cq;
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
            float *d0 = a.dq + (r * a.H + h0 + mm * 16 + gq) * (int64_t)DQK + col;
            *reinterpret_cast<float2 *>(d0) = make_float2(dq[j][mm][0], dq[j][mm][1]);
            *reinterpret_cast<float2 *>(d0 + 8 * DQK) = make_float2(dq[j][mm][2], dq[j][mm][3]);
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
