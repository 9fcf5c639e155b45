// score_tc.cu -- Lightning Indexer scores on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA, for the streaming (decode / hierarchical) scoring passes.
//
// Paper: Sec. 2.2 Eq. 1  I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]);  Sec. 3.3 Eq. 9 (page
// score over sub-block-mean keys) and Eq. 10 (stage-2 token scores in the recalled pages).
//
// Shape of the contraction: per query row, D[key, head] = sum_d k[key, d] * q[head, d] with
// the keys as the MMA's M = 128 rows, the H_I heads as N and d_I as K.  One TMEM accumulator row
// then holds all head logits of one key, so ReLU, the head weights and the head sum are
// thread-local in the epilogue (no shuffles, no shared-memory transpose).
//
// Warp roles (192 threads; 320 for the FP8 scorer at 64 heads, which adds a second epilogue
// group in warps 6-9 taking every other tile from four TMEM accumulators):
//   warps 0-3  epilogue: tcgen05.ld of the 128 x H_I fp32 tile (warp w reads TMEM lanes
//              32w..32w+31 = keys), score = sum_j w_j max(x_j, 0), store the fp32 score, bump the
//              CTA's shared-memory histogram of the score's top 12 key bits (used by the top-K);
//   warp 4     TMA producer: 128-row key tiles (two 64-column SWIZZLE_128B boxes for d_I = 128)
//              into a ring of shared-memory stages;
//   warp 5     TMEM allocator and MMA issuer: one elected thread issues K/16 tcgen05.mma per tile
//              into one of two TMEM accumulators and commits to the stage's "empty" barrier and
//              the accumulator's "full" barrier.
// Every wait is bounded (about 4 s); on expiry the CTA raises LSA_DEVERR_TIMEOUT, stops issuing,
// drains what it issued and frees its TMEM.
//
// Each CTA owns one contiguous chunk of tiles of one query row (grid = chunks x rows).  Shared
// memory ~ 97 KB so two CTAs share an SM and one CTA's prologue hides behind the other's stream.
//
// FP8 variant (F8 = true, tokens mode, d_I = 128): keys and queries are E4M3 codes, one 128-byte
// SWIZZLE_128B row each, and the MMA is kind::f8f6f4 with K = 32 per instruction (the same four
// 32-byte k-steps per row as bf16).  The per-(query, head) scales are folded into the head
// weights and the per-key scale multiplies the head sum (both are positive, so they commute with
// the ReLU): score = ks[key] * sum_j (w_j qs_j) max(acc_j, 0).
#include <cuda.h>

#include "lsa_internal.cuh"
#include "score_tc.cuh"
#include "score_common.cuh"
#include "select_util.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace tc;

constexpr int kTile = 128;       // keys (M) per tile
// TMA ring depth: bf16 tiles are 32 KB (d_I = 128), FP8 tiles 16 KB.  Both run two CTAs per SM;
// bf16 with two stages, FP8 with four (about 90 KB of shared memory and, at 64 heads, 256 TMEM
// columns each), so that half the bytes per tile still keep as many bytes in flight per SM
template <bool F8>
__host__ __device__ constexpr int stages_of() { return F8 ? 4 : 2; }
// Epilogue warpgroups: FP8 with 64 heads runs two, each taking every other tile, over four TMEM
// accumulators, so that two tiles' epilogues overlap in a CTA (the per-tile epilogue, not the
// tile's bytes, sets the rate of one warpgroup).
template <bool F8, int N>
__host__ __device__ constexpr int epi_groups() { return (F8 && N == 64) ? 2 : 1; }
template <bool F8, int N>
__host__ __device__ constexpr int threads_of() { return 64 + 128 * epi_groups<F8, N>(); }

// Shared-memory plan (offsets from a 1024-aligned base).
template <int N, int KC, int kStages>
struct Smem {
    static constexpr int kQ = 0;                                 // KC x N x 128 B
    static constexpr int kKeys = kQ + KC * N * 128;              // stages x KC x 16 KB
    static constexpr int kStageBytes = KC * kTile * 128;
    static constexpr int kHist = kKeys + kStages * kStageBytes;  // 4096 x u32
    static constexpr int kW = kHist + kHistBins * 4;             // N floats
    static constexpr int kBars = kW + N * 4;                     // 2*stages + 9 barriers
    static constexpr int kMisc = kBars + (2 * kStages + 9) * 8;  // tmem addr, abort flag
    static constexpr int kTotal = kMisc + 16;
};

// Element-wise max(x, 0) (POS) or min(x, 0) of eight packed bf16 values (exact: each result is
// one of the inputs or zero).
template <bool POS>
__device__ __forceinline__ uint4 clamp_bf16x8(uint4 v) {
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&w[i]);
        const __nv_bfloat162 z = __float2bfloat162_rn(0.f);
        x = POS ? __hmax2(x, z) : __hmin2(x, z);
        w[i] = *reinterpret_cast<uint32_t *>(&x);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// MM (MinMax pooling, pages mode): the key rows are (k_max | k_min) of 2 d_I dims and the query
// operand is (max(q, 0) | min(q, 0)), so one contraction of depth 2 d_I gives
// sum_d max(q_d k_max_d, q_d k_min_d) = q+ . k_max + q- . k_min for every head.
// Resident CTAs per SM the launch plans for (registers are capped so that they fit).
template <bool F8, int N>
__host__ __device__ constexpr int ctas_per_sm() { return 2; }

template <int N, int KC, bool F8, bool MM>
__global__ void __launch_bounds__(threads_of<F8, N>(), ctas_per_sm<F8, N>())
    score_tc_kernel(const __grid_constant__ CUtensorMap keymap, TcScoreArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    constexpr int kStages = stages_of<F8>();
    constexpr int kThreads = threads_of<F8, N>();
    constexpr int EG = epi_groups<F8, N>();
    constexpr int NACC = 2 * EG;  // TMEM accumulators
    using S = Smem<N, KC, kStages>;
    uint8_t *q_s = sm + S::kQ;
    uint8_t *keys_s = sm + S::kKeys;
    uint32_t *hist_s = reinterpret_cast<uint32_t *>(sm + S::kHist);
    float *w_s = reinterpret_cast<float *>(sm + S::kW);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + S::kBars);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;  // [NACC]
    uint64_t *tempty = tfull + NACC;    // [NACC]
    uint64_t *drain = tempty + NACC;    // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + S::kMisc + 4);
    __shared__ uint32_t scratch[40];
    __shared__ int s_last;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t r = blockIdx.y;
    const int64_t b = r / a.T;
    const int64_t t = a.q_pos[r];
    const int64_t len = a.kv_len[b];
    if (!(t >= 0 && t < len && len <= a.L_max)) {
        if (blockIdx.x == 0 && tid == 0) raise_error(a.err, LSA_DEVERR_QPOS);
        return;
    }
    const Regions g = regions_of(t, a.Ks, a.Kw);
    // units of this row: tokens of dyn / sub-blocks of the eligible pages / recalled tokens
    int64_t u_lo = 0, n_units = 0, p0 = 0, p1 = 0, nb = 0;
    const int G = a.P / a.Bsub;  // sub-blocks per page (pages mode)
    if (a.mode == kScoreTokens) {
        u_lo = g.dyn_lo;
        n_units = g.dyn_hi - g.dyn_lo;
    } else if (a.mode == kScorePages) {
        if (g.dyn_hi > g.dyn_lo) {
            p0 = g.dyn_lo / a.P;
            p1 = (g.dyn_hi - 1) / a.P + 1;
            nb = (len + a.Bsub - 1) / a.Bsub;
            u_lo = p0 * G;
            int64_t u_hi = p1 * G;
            if (u_hi > nb) u_hi = nb;
            n_units = u_hi - u_lo;
        }
    } else {
        n_units = (int64_t)a.page_count[r] * kTile;
    }
    const int64_t n_tiles = (n_units + kTile - 1) / kTile;
    const int64_t tile0 = (int64_t)blockIdx.x * a.chunk_tiles;
    int64_t tile1 = tile0 + a.chunk_tiles;
    if (tile1 > n_tiles) tile1 = n_tiles;
    if (tile0 >= tile1) {
        if (a.hist) row_done(a, r, hist_s, scratch, &s_last);
        return;
    }
    const int n_my = (int)(tile1 - tile0);

    // ---- set-up: q (SWIZZLE_128B, K-major), w, histogram, barriers, TMEM
    {
        // bytes of one query row's q: QC chunks of 128 B per head (MinMax reads each twice)
        constexpr int QC = MM ? KC / 2 : KC;
        const uint8_t *qr = F8 ? a.q8 + r * (int64_t)N * 128
                               : reinterpret_cast<const uint8_t *>(a.q + r * (int64_t)N * (QC * 64));
        // chunk c (16 B) of row h in k-chunk kc lands at kc*N*128 + h*128 + ((c ^ (h & 7)) * 16)
        for (int i = tid; i < KC * N * 8; i += kThreads) {
            const int kc = i / (N * 8), rem = i - kc * N * 8, h = rem >> 3, c = rem & 7;
            uint4 v = *reinterpret_cast<const uint4 *>(qr + h * (QC * 128) + (kc % QC) * 128 + c * 16);
            if (MM) v = kc < QC ? clamp_bf16x8<true>(v) : clamp_bf16x8<false>(v);
            *reinterpret_cast<uint4 *>(q_s + kc * N * 128 + h * 128 + ((c ^ (h & 7)) << 4)) = v;
        }
        for (int j = tid; j < N; j += kThreads)
            w_s[j] = F8 ? __bfloat162float(a.w[r * N + j]) * a.qscale[r * N + j]
                        : __bfloat162float(a.w[r * N + j]);
        if (a.hist)
            for (int i = tid; i < kHistBins; i += kThreads) hist_s[i] = 0;
        if (tid == 0) {
            for (int s = 0; s < kStages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            for (int s = 0; s < NACC; ++s) {
                mbar_init(&tfull[s], 1);
                mbar_init(&tempty[s], 128);
            }
            mbar_init(drain, 1);
            *abort = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        if (warp == 5) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32(tmem_slot)), "r"(NACC * N));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // q visible to the MMA
        fence_before();
        __syncthreads();
        fence_after();
    }
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const int64_t seq_rows = (a.mode == kScorePages) ? a.nb_max : a.L_max;
            int issued = 0;
            // stage 2: the page of tile k is read one tile ahead, so that its global-load latency
            // overlaps the wait for a free stage instead of delaying the tile's copy
            // (the FP8 scorer has no stage-2 mode)
            const int32_t *pages =
                (!F8 && a.mode == kScoreStage2) ? a.page_list + r * a.page_stride : nullptr;
            int64_t pg_next = pages ? (int64_t)pages[tile0] : 0;
            for (int k = 0; k < n_my; ++k) {
                const int s = k % kStages;
                if (k >= kStages && !mbar_wait(&empty[s], ((k / kStages) & 1) ^ 1, abort, a.err))
                    break;
                const int64_t tl = tile0 + k;
                int64_t row0;
                if (pages) {
                    row0 = pg_next * kTile;
                    if (k + 1 < n_my) pg_next = (int64_t)pages[tl + 1];
                } else {
                    row0 = u_lo + tl * kTile;
                }
                const int y = (int)(b * seq_rows + row0);
                mbar_expect_tx(&full[s], S::kStageBytes);
                for (int kc = 0; kc < KC; ++kc)
                    tma_load_2d(keys_s + s * S::kStageBytes + kc * kTile * 128, &keymap, kc * 64, y,
                                &full[s]);
                ++issued;
            }
            if (*abort) {
                // drain the copies still in flight before the CTA may exit
                for (int k = (issued > kStages ? issued - kStages : 0); k < issued; ++k) {
                    const int s = k % kStages;
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try(&full[s], (k / kStages) & 1))
                        if (globaltimer() - t0 > kWaitNs) break;
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // kind::f16: D f32, A/B bf16 (formats 1); kind::f8f6f4: A/B E4M3 (formats 0); both
            // K-major, N, M = 128
            const uint32_t idesc = (1u << 4) | (F8 ? 0u : (1u << 7) | (1u << 10)) |
                                   ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kTile >> 4) << 24);
            const uint32_t q_addr = smem_u32(q_s);
            const uint32_t k_addr = smem_u32(keys_s);
            for (int k = 0; k < n_my; ++k) {
                const int s = k % kStages, acc = k % NACC;
                if (!mbar_wait(&full[s], (k / kStages) & 1, abort, a.err)) break;
                if (k >= NACC && !mbar_wait(&tempty[acc], ((k / NACC) & 1) ^ 1, abort, a.err))
                    break;
                fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * N);
#pragma unroll
                for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t ad =
                            sw128_desc(k_addr + s * S::kStageBytes + kc * kTile * 128 + ks * 32);
                        const uint64_t bd = sw128_desc(q_addr + kc * N * 128 + ks * 32);
                        if (F8)
                            umma_e4m3(d_tmem, ad, bd, idesc, (kc | ks) != 0);
                        else
                            umma_bf16(d_tmem, ad, bd, idesc, (kc | ks) != 0);
                    }
                }
                umma_commit(&empty[s]);
                umma_commit(&tfull[acc]);
            }
            // wait until every MMA this thread issued has completed
            umma_commit(drain);
            const uint64_t t0 = globaltimer();
            while (!mbar_try(drain, 0))
                if (globaltimer() - t0 > kWaitNs) {
                    raise_error(a.err, LSA_DEVERR_TIMEOUT);
                    break;
                }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 0-3, and
        // 6-9 for a second group): group eg takes the tiles k = eg, eg + EG, ...
        const int eg = warp >= 6 ? 1 : 0, quad = warp & 3;
        const int row_in_tile = quad * 32 + lane;  // TMEM lane = key row of the tile
        float *out = a.out + r * a.out_stride;
        bool nonfinite = false;
        // FP8: this tile's key scale is loaded one tile ahead, so its global-load latency
        // overlaps the wait for the accumulator instead of following it
        auto key_scale = [&](int kk) -> float {
            const int64_t u = (tile0 + kk) * kTile + row_in_tile;
            return u < n_units ? __ldg(a.kscale + b * a.L_max + u_lo + u) : 0.f;
        };
        float ks_cur = (F8 && eg < n_my) ? key_scale(eg) : 0.f;
        // stage 2: the tile's page, read one tile ahead for the same reason
        auto page_of = [&](int kk) -> int64_t {
            return (!F8 && a.mode == kScoreStage2 && kk < n_my)
                       ? (int64_t)a.page_list[r * a.page_stride + tile0 + kk] : 0;
        };
        int64_t pg_cur = page_of(eg);
        for (int k = eg; k < n_my; k += EG) {
            const int acc = k % NACC;
            const float ks_next = (F8 && k + EG < n_my) ? key_scale(k + EG) : 0.f;
            const int64_t pg_next = page_of(k + EG);
            // the TMEM loads below are warp-collective: leave the loop only as a whole warp
            // (lane 0 alone polls the barrier, so that the epilogue warps of the CTAs on an SM
            // do not crowd the shared-memory port the TMA and the tensor core use)
            if (!warp_wait(&tfull[acc], (k / NACC) & 1, abort, a.err)) break;
            fence_after();
            // four independent partial sums over the heads (a 64-long dependent FMA chain would
            // cost 64 FMA latencies per tile), added at the end
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
            for (int c = 0; c < N / 64; ++c) {
                uint32_t v[64];
                tmem_ld64(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * N + c * 64), v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 64; j += 4) {
                    const float4 wv = *reinterpret_cast<const float4 *>(w_s + c * 64 + j);
                    s0 = fmaf(wv.x, fmaxf(__uint_as_float(v[j]), 0.f), s0);
                    s1 = fmaf(wv.y, fmaxf(__uint_as_float(v[j + 1]), 0.f), s1);
                    s2 = fmaf(wv.z, fmaxf(__uint_as_float(v[j + 2]), 0.f), s2);
                    s3 = fmaf(wv.w, fmaxf(__uint_as_float(v[j + 3]), 0.f), s3);
                }
            }
            float score = (s0 + s1) + (s2 + s3);
            fence_before();
            mbar_arrive(&tempty[acc]);
            const int64_t tl = tile0 + k;
            const int64_t u = tl * kTile + row_in_tile;  // unit index within the row
            if (a.mode == kScoreTokens) {
                uint32_t key = 0;
                if (u < n_units) {
                    const int64_t pos = u_lo + u;
                    if (F8) score *= ks_cur;
                    out[pos] = score;
                    nonfinite |= !isfinite(score);
                    key = order_key(score);
                }
                if (a.hist) hist_add_warp(hist_s, key);
            } else if (a.mode == kScoreStage2) {
                const int64_t pos = pg_cur * kTile + row_in_tile;
                uint32_t key = 0;
                if (pos >= g.dyn_lo && pos < g.dyn_hi) {
                    out[u] = score;
                    nonfinite |= !isfinite(score);
                    key = order_key(score);
                } else {
                    out[u] = excluded_score();
                }
                if (a.hist) hist_add_warp(hist_s, key);
            } else {
                // pages: sum G consecutive sub-block scores (G divides 32)
                float ps = (u < n_units) ? score : 0.f;
                for (int o = G >> 1; o > 0; o >>= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, o);
                const int64_t sb = u_lo + u;  // sub-block id
                uint32_t key = 0;
                if ((lane & (G - 1)) == 0 && u < n_units) {
                    const int64_t page = sb / G;
                    if (page < p1) {
                        out[page] = ps;
                        nonfinite |= !isfinite(ps);
                        key = order_key(ps);
                    }
                }
                if (a.hist) hist_add_warp(hist_s, key);
            }
            ks_cur = ks_next;
            pg_cur = pg_next;
        }
        if (nonfinite) raise_error(a.err, LSA_DEVERR_NONFINITE);
    }

    // ---- tear-down: flush the histogram, free TMEM
    fence_before();
    __syncthreads();
    fence_after();
    if (a.hist) {
        uint32_t *gh = a.hist + r * kHistBins;
        for (int i = tid; i < kHistBins; i += kThreads) {
            const uint32_t v = hist_s[i];
            if (v) atomicAdd(&gh[i], v);
        }
    }
    if (warp == 5) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(NACC * N));
    }
    if (a.hist) row_done(a, r, hist_s, scratch, &s_last);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

template <int N, int KC, bool F8 = false, bool MM = false>
cudaError_t launch_tc(const CUtensorMap &map, const TcScoreArgs &a, int64_t rows,
                      cudaStream_t s) {
    using S = Smem<N, KC, stages_of<F8>()>;
    const int smem = S::kTotal + 1024;
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<N, KC, F8, MM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // the whole unified L1 / shared-memory array as shared memory, so that the planned number of
    // CTAs fits on an SM
    e = cudaFuncSetAttribute(score_tc_kernel<N, KC, F8, MM>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.n_chunks, (unsigned)rows);
    score_tc_kernel<N, KC, F8, MM><<<grid, threads_of<F8, N>(), smem, s>>>(map, a);
    return launched();
}

// chunks per row so that the grid is about per_sm CTAs per SM (one wave)
void set_chunks(TcScoreArgs &a, int64_t rows, int64_t max_tiles, int per_sm = 2) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t chunks = ((int64_t)per_sm * sms) / rows;
    if (chunks < 1) chunks = 1;
    if (chunks > max_tiles) chunks = max_tiles;
    a.chunk_tiles = (int)((max_tiles + chunks - 1) / chunks);
    a.n_chunks = (int)((max_tiles + a.chunk_tiles - 1) / a.chunk_tiles);
}

}  // namespace

bool make_tmap_2d_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                       uint32_t box_inner, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)inner * 2};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), gdim, gstride,
              box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_2d_u8(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                     uint32_t box_inner, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)inner};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), gdim, gstride,
              box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_score_supported(int H, int D, int mode, int P, int Bsub, int64_t key_rows) {
    if (!(H == 64 || H == 128) || !(D == 64 || D == 128)) return false;
    if (key_rows <= 0 || key_rows >= 0x7FFFFFFFll) return false;
    if (mode == kScoreStage2 && P != kTile) return false;
    if (mode == kScorePages) {
        const int G = P / Bsub;
        if (G < 1 || G > 32 || (G & (G - 1))) return false;
    }
    return encode_fn() != nullptr;
}

cudaError_t launch_score_tc(const TcScoreArgs &a0, const void *keys, int64_t key_rows, int D,
                            int64_t rows, int64_t max_tiles, cudaStream_t s) {
    if (rows <= 0 || max_tiles <= 0) return cudaSuccess;
    if (rows > 65535) return cudaErrorInvalidValue;
    TcScoreArgs a = a0;
    set_chunks(a, rows, max_tiles);

    CUtensorMap map;
    const int H = a.H;
    if (a.minmax) {
        // MinMax pooling rows (k_max | k_min): 2 D dims per sub-block
        if (a.mode != kScorePages) return cudaErrorInvalidValue;
        if (!make_tmap_2d_bf16(&map, keys, (uint64_t)(2 * D), (uint64_t)key_rows, 64, kTile))
            return cudaErrorInvalidValue;
        if (H == 64 && D == 128) return launch_tc<64, 4, false, true>(map, a, rows, s);
        if (H == 128 && D == 128) return launch_tc<128, 4, false, true>(map, a, rows, s);
        if (H == 64 && D == 64) return launch_tc<64, 2, false, true>(map, a, rows, s);
        if (H == 128 && D == 64) return launch_tc<128, 2, false, true>(map, a, rows, s);
        return cudaErrorInvalidValue;
    }
    if (!make_tmap_2d_bf16(&map, keys, (uint64_t)D, (uint64_t)key_rows, 64, kTile))
        return cudaErrorInvalidValue;
    if (H == 64 && D == 128) return launch_tc<64, 2>(map, a, rows, s);
    if (H == 128 && D == 128) return launch_tc<128, 2>(map, a, rows, s);
    if (H == 64 && D == 64) return launch_tc<64, 1>(map, a, rows, s);
    if (H == 128 && D == 64) return launch_tc<128, 1>(map, a, rows, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_score_tc_fp8(const TcScoreArgs &a0, const void *keys8, int64_t key_rows, int D,
                                int64_t rows, int64_t max_tiles, cudaStream_t s) {
    if (rows <= 0 || max_tiles <= 0) return cudaSuccess;
    if (rows > 65535 || D != 128 || a0.mode != kScoreTokens) return cudaErrorInvalidValue;
    TcScoreArgs a = a0;
    set_chunks(a, rows, max_tiles, a.H == 64 ? ctas_per_sm<true, 64>() : ctas_per_sm<true, 128>());
    CUtensorMap map;
    if (!make_tmap_2d_u8(&map, keys8, (uint64_t)D, (uint64_t)key_rows, 128, kTile))
        return cudaErrorInvalidValue;
    if (a.H == 64) return launch_tc<64, 1, true>(map, a, rows, s);
    if (a.H == 128) return launch_tc<128, 1, true>(map, a, rows, s);
    return cudaErrorInvalidValue;
}

}  // namespace lsa
