// score_mq.cu -- Lightning Indexer scores of several queries of one sequence per CTA on the
// 5th-generation tensor cores (prefill: the T > 1 queries of a chunk share the key cache).
//
// Paper: Sec. 2.2 Eq. 1  I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]) over the dynamic region of
// Sec. 3.1; Sec. 4.1.2 and Table 4 (the prefill indexer is an O(L^2) contraction).
//
// Shape: one CTA scores G consecutive queries of one sequence against a contiguous chunk of
// 128-key tiles: D[key, (g, head)] = sum_d k[key, d] * q[g, head, d], with the keys as the MMA's
// M = 128 rows, the G x H_I query heads as N = 256 and d_I = 128 as K.  Every key tile streamed
// from L2 then feeds G queries (the one-query kernel fetches it once per query), and each MMA is
// N = 256 wide, which the tensor core runs at its full rate (an M = 128, K = 16 MMA costs about
// the same to issue for any N up to 128).  The two TMEM accumulators take all 512 columns, so
// one CTA runs per SM.
//
// Warp roles (320 threads):
//   warps 0-7  epilogue: warp w reads TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31 (the tile's keys)
//              of the columns of queries (w / 4) * G/2 .. (w / 4 + 1) * G/2 - 1; score =
//              sum_j w_j max(x_j, 0), stored when the key lies in that query's dyn and counted in
//              that query's shared-memory histogram of the score's top 12 key bits;
//   warp 8     TMA producer: 128-key tiles (two 64-column SWIZZLE_128B boxes) into a 3-stage ring;
//   warp 9     TMEM allocator and single-thread MMA issuer.
// Every wait is bounded; on expiry the CTA raises LSA_DEVERR_TIMEOUT, stops issuing, drains what
// it issued and frees its TMEM.  A query outside its sequence raises LSA_DEVERR_QPOS and takes no
// part (its row is skipped by the selection).
#include <cuda.h>

#include "lsa_internal.cuh"
#include "score_common.cuh"
#include "score_tc.cuh"
#include "select_util.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace tc;

constexpr int kTile = 128;      // keys (M) per tile
constexpr int kStages = 3;      // 32 KB key tiles
constexpr int KC = 2;           // 64-dim chunks of d_I = 128
constexpr int N = 256;          // G x H_I accumulator columns
constexpr int kEpiWarps = 8;
constexpr int kProdWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kThreads = 32 * (kMmaWarp + 1);

template <int G>
struct SmemMq {
    static constexpr int kQ = 0;                                   // KC x N x 128 B
    static constexpr int kKeys = kQ + KC * N * 128;                // stages x KC x 16 KB
    static constexpr int kStageBytes = KC * kTile * 128;
    static constexpr int kHist = kKeys + kStages * kStageBytes;    // G x 4096 x u32
    static constexpr int kW = kHist + G * kHistBins * 4;           // N floats
    static constexpr int kBars = kW + N * 4;                       // 2 stages + 5 barriers
    static constexpr int kMisc = kBars + (2 * kStages + 5) * 8;    // tmem addr, abort flag
    static constexpr int kTotal = kMisc + 16;
};

// x[g] for a g known only at run time, without indexing the register array (which would put
// it in local memory)
template <int G, typename T>
__device__ __forceinline__ T pick(const T (&x)[G], int g) {
    T v = x[0];
#pragma unroll
    for (int i = 1; i < G; ++i)
        if (g == i) v = x[i];
    return v;
}

// PAGES (HI stage 1, Eq. 9): the units are the sub-block means of the sequence; a query's units
// are the sub-blocks of the pages that intersect its dyn (those present), and each page's score
// is the sum of its Gs = P / B_sub consecutive sub-block scores (a shuffle over Gs lanes).
template <int H, int G, bool PAGES>
__global__ void __launch_bounds__(kThreads, 1)
    score_mq_kernel(const __grid_constant__ CUtensorMap keymap, TcScoreArgs a, int groups_per_seq) {
    static_assert(G * H == N, "G queries x H heads fill the 256 accumulator columns");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    using S = SmemMq<G>;
    uint8_t *q_s = sm + S::kQ;
    uint8_t *keys_s = sm + S::kKeys;
    uint32_t *hist_s = reinterpret_cast<uint32_t *>(sm + S::kHist);  // [G][kHistBins]
    float *w_s = reinterpret_cast<float *>(sm + S::kW);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + S::kBars);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;  // [2]
    uint64_t *tempty = tfull + 2;       // [2]
    uint64_t *drain = tempty + 2;       // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + S::kMisc + 4);
    __shared__ uint32_t scratch[40];
    __shared__ int s_last;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the group: G consecutive queries of sequence b (the last group of a sequence may be short)
    const int64_t b = blockIdx.y / groups_per_seq;
    const int64_t tq0 = (int64_t)(blockIdx.y % groups_per_seq) * G;
    const int64_t len = a.kv_len[b];
    // units of query g: [u_lo, his[g]); tokens: its dyn; pages: the present sub-blocks of the
    // pages intersecting its dyn, whose ends page_end[g] bound the pages it scores
    int64_t rows[G], his[G], page_end[G];
    bool valid[G];
    const int Gs = PAGES ? a.P / a.Bsub : 1;            // sub-blocks per page
    const int64_t nb = (len + a.Bsub - 1) / a.Bsub;     // sub-blocks present (pages)
    const int64_t u_lo = PAGES ? (int64_t)(a.Ks / a.P) * Gs : a.Ks;  // every dyn starts at Ks
    int64_t u_hi = u_lo;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        rows[g] = b * a.T + tq0 + g;
        his[g] = u_lo;
        page_end[g] = 0;
        valid[g] = false;
        if (tq0 + g >= a.T) continue;
        const int64_t t = a.q_pos[rows[g]];
        if (!(t >= 0 && t < len && len <= a.L_max)) {
            if (blockIdx.x == 0 && tid == 0) raise_error(a.err, LSA_DEVERR_QPOS);
            continue;
        }
        valid[g] = true;
        const Regions rg = regions_of(t, a.Ks, a.Kw);
        if (rg.dyn_hi > rg.dyn_lo) {
            if (PAGES) {
                page_end[g] = (rg.dyn_hi - 1) / a.P + 1;
                his[g] = min(page_end[g] * Gs, nb);
            } else {
                his[g] = rg.dyn_hi;
            }
        }
        if (his[g] > u_hi) u_hi = his[g];
    }
    bool any_valid = false;
#pragma unroll
    for (int g = 0; g < G; ++g) any_valid |= valid[g];
    if (!any_valid) return;
    const int64_t n_units = u_hi > u_lo ? u_hi - u_lo : 0;
    const int64_t n_tiles = (n_units + kTile - 1) / kTile;
    const int64_t tile0 = (int64_t)blockIdx.x * a.chunk_tiles;
    int64_t tile1 = tile0 + a.chunk_tiles;
    if (tile1 > n_tiles) tile1 = n_tiles;
    auto finish_rows = [&]() {
#pragma unroll
        for (int g = 0; g < G; ++g)
            if (valid[g] && a.hist) row_done(a, rows[g], hist_s, scratch, &s_last);
    };
    if (tile0 >= tile1) {
        finish_rows();
        return;
    }
    const int n_my = (int)(tile1 - tile0);

    // ---- set-up: q of the G queries (SWIZZLE_128B, K-major: accumulator column g*H + j is
    // query g's head j), head weights, histograms, barriers, TMEM
    {
        // chunk c (16 B) of row n in k-chunk kc lands at kc*N*128 + n*128 + ((c ^ (n & 7)) * 16)
        for (int i = tid; i < KC * N * 8; i += kThreads) {
            const int kc = i / (N * 8), rem = i - kc * N * 8, n = rem >> 3, c = rem & 7;
            const int g = n / H, j = n - g * H;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (pick(valid, g))
                v = *reinterpret_cast<const uint4 *>(
                    reinterpret_cast<const uint8_t *>(a.q + (pick(rows, g) * H + j) *
                                                                (int64_t)(KC * 64)) +
                    kc * 128 + c * 16);
            *reinterpret_cast<uint4 *>(q_s + kc * N * 128 + n * 128 + ((c ^ (n & 7)) << 4)) = v;
        }
        for (int n = tid; n < N; n += kThreads) {
            const int g = n / H, j = n - g * H;
            w_s[n] = pick(valid, g) ? __bfloat162float(a.w[pick(rows, g) * H + j]) : 0.f;
        }
        if (a.hist)
            for (int i = tid; i < G * kHistBins; i += kThreads) hist_s[i] = 0;
        if (tid == 0) {
            for (int s = 0; s < kStages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            for (int s = 0; s < 2; ++s) {
                mbar_init(&tfull[s], 1);
                mbar_init(&tempty[s], 32 * kEpiWarps);
            }
            mbar_init(drain, 1);
            *abort = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        if (warp == kMmaWarp) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32(tmem_slot)), "r"(2 * N));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // q visible to the MMA
        fence_before();
        __syncthreads();
        fence_after();
    }
    const uint32_t tmem = *tmem_slot;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int k = 0; k < n_my; ++k) {
                const int s = k % kStages;
                if (k >= kStages && !mbar_wait(&empty[s], ((k / kStages) & 1) ^ 1, abort, a.err))
                    break;
                const int64_t row0 = u_lo + (tile0 + k) * kTile;
                const int y = (int)(b * (PAGES ? a.nb_max : a.L_max) + row0);
                mbar_expect_tx(&full[s], S::kStageBytes);
#pragma unroll
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
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // kind::f16: D f32, A/B bf16, both K-major; N = 256, M = 128
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                   ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kTile >> 4) << 24);
            const uint32_t q_addr = smem_u32(q_s);
            const uint32_t k_addr = smem_u32(keys_s);
            for (int k = 0; k < n_my; ++k) {
                const int s = k % kStages, acc = k & 1;
                if (!mbar_wait(&full[s], (k / kStages) & 1, abort, a.err)) break;
                if (k >= 2 && !mbar_wait(&tempty[acc], ((k >> 1) & 1) ^ 1, abort, a.err)) break;
                fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * N);
#pragma unroll
                for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t ad =
                            sw128_desc(k_addr + s * S::kStageBytes + kc * kTile * 128 + ks * 32);
                        const uint64_t bd = sw128_desc(q_addr + kc * N * 128 + ks * 32);
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
        // ------------------------------------------------------------ epilogue (warps 0-7)
        constexpr int GW = G / 2;                // queries per warp
        const int quarter = warp & 3, half = warp >> 2;
        bool my_valid[GW];
        int64_t my_row[GW], my_hi[GW], my_pend[GW];
#pragma unroll
        for (int gg = 0; gg < GW; ++gg) {
            my_valid[gg] = pick(valid, half * GW + gg);
            my_row[gg] = pick(rows, half * GW + gg);
            my_hi[gg] = pick(his, half * GW + gg);
            my_pend[gg] = pick(page_end, half * GW + gg);
        }
        const int row_in_tile = quarter * 32 + lane;  // TMEM lane = key row of the tile
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        bool nonfinite = false;
        for (int k = 0; k < n_my; ++k) {
            const int acc = k & 1;
            // the TMEM loads below are warp-collective: leave the loop only as a whole warp
            if (!warp_wait(&tfull[acc], (k >> 1) & 1, abort, a.err)) break;
            fence_after();
            float score[GW];
#pragma unroll
            for (int gg = 0; gg < GW; ++gg) {
                const int g = half * GW + gg;
                // four independent partial sums over the heads
                float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
                for (int c = 0; c < H / 64; ++c) {
                    uint32_t v[64];
                    tmem_ld64(tmem + lane_base + (uint32_t)(acc * N + g * H + c * 64), v);
                    tmem_wait_ld();
                    const float *wg = w_s + g * H + c * 64;
#pragma unroll
                    for (int j = 0; j < 64; j += 4) {
                        const float4 wv = *reinterpret_cast<const float4 *>(wg + j);
                        s0 = fmaf(wv.x, fmaxf(__uint_as_float(v[j]), 0.f), s0);
                        s1 = fmaf(wv.y, fmaxf(__uint_as_float(v[j + 1]), 0.f), s1);
                        s2 = fmaf(wv.z, fmaxf(__uint_as_float(v[j + 2]), 0.f), s2);
                        s3 = fmaf(wv.w, fmaxf(__uint_as_float(v[j + 3]), 0.f), s3);
                    }
                }
                score[gg] = (s0 + s1) + (s2 + s3);
            }
            fence_before();
            mbar_arrive(&tempty[acc]);
            const int64_t pos = u_lo + (tile0 + k) * kTile + row_in_tile;  // token or sub-block
#pragma unroll
            for (int gg = 0; gg < GW; ++gg) {
                const int g = half * GW + gg;
                uint32_t key = 0;
                if (PAGES) {
                    // page score: the sum of its Gs sub-blocks (those present); Gs divides 32
                    float ps = (my_valid[gg] && pos < my_hi[gg]) ? score[gg] : 0.f;
                    for (int o = Gs >> 1; o > 0; o >>= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, o);
                    const int64_t page = pos / Gs;
                    if ((lane & (Gs - 1)) == 0 && my_valid[gg] && pos < my_hi[gg] &&
                        page < my_pend[gg]) {
                        a.out[my_row[gg] * a.out_stride + page] = ps;
                        nonfinite |= !isfinite(ps);
                        key = order_key(ps);
                    }
                } else if (my_valid[gg] && pos < my_hi[gg]) {
                    a.out[my_row[gg] * a.out_stride + pos] = score[gg];
                    nonfinite |= !isfinite(score[gg]);
                    key = order_key(score[gg]);
                }
                if (a.hist) hist_add_warp(hist_s + g * kHistBins, key);
            }
        }
        if (nonfinite) raise_error(a.err, LSA_DEVERR_NONFINITE);
    }

    // ---- tear-down: flush the histograms, free TMEM, then the per-row threshold step
    fence_before();
    __syncthreads();
    fence_after();
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (!valid[g] || !a.hist) continue;
        uint32_t *gh = a.hist + rows[g] * kHistBins;
        const uint32_t *hs = hist_s + g * kHistBins;
        for (int i = tid; i < kHistBins; i += kThreads) {
            const uint32_t v = hs[i];
            if (v) atomicAdd(&gh[i], v);
        }
    }
    if (warp == kMmaWarp) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(2 * N));
    }
    finish_rows();
}

template <int H, int G, bool PAGES>
cudaError_t launch_mq(const CUtensorMap &map, const TcScoreArgs &a, int groups_per_seq,
                      int64_t n_groups, cudaStream_t s) {
    using S = SmemMq<G>;
    const int smem = S::kTotal + 1024;
    cudaError_t e = cudaFuncSetAttribute(score_mq_kernel<H, G, PAGES>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.n_chunks, (unsigned)n_groups);
    score_mq_kernel<H, G, PAGES><<<grid, kThreads, smem, s>>>(map, a, groups_per_seq);
    return launched();
}

static_assert(SmemMq<4>::kTotal + 1024 <= 232448, "shared memory plan exceeds 227 KB");

}  // namespace

bool mq_score_supported(int H, int D, int T, int mode, int P, int Bsub, int minmax) {
    if (!((H == 64 || H == 128) && D == 128 && T >= 2 && !minmax)) return false;
    if (mode == kScoreTokens) return true;
    if (mode != kScorePages || Bsub < 1) return false;
    const int Gs = P / Bsub;
    return Gs >= 1 && Gs <= 32 && (Gs & (Gs - 1)) == 0;
}

cudaError_t launch_score_mq(const TcScoreArgs &a0, const void *keys, int64_t key_rows, int B,
                            int64_t max_tiles, cudaStream_t s) {
    if (B <= 0 || max_tiles <= 0) return cudaSuccess;
    TcScoreArgs a = a0;
    const int G = N / a.H;
    const int groups_per_seq = (a.T + G - 1) / G;
    const int64_t n_groups = (int64_t)B * groups_per_seq;
    if (n_groups > 65535 || (a.mode != kScoreTokens && a.mode != kScorePages))
        return cudaErrorInvalidValue;
    // key chunks per group: fill the SMs (one CTA each) with the least idle tail of the last wave
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t best = 1;
    double best_eff = -1.0;
    for (int64_t c = 1; c <= 16 && c <= max_tiles; ++c) {
        const int64_t ctas = n_groups * c;
        const int64_t waves = (ctas + sms - 1) / sms;
        // fraction of the launched SM-waves doing work, less a small cost per extra chunk
        const double eff = (double)ctas / (double)(waves * sms) - 0.01 * (double)(c - 1);
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best = c;
        }
    }
    a.chunk_tiles = (int)((max_tiles + best - 1) / best);
    a.n_chunks = (int)((max_tiles + a.chunk_tiles - 1) / a.chunk_tiles);
    CUtensorMap map;
    if (!make_tmap_2d_bf16(&map, keys, 128, (uint64_t)key_rows, 64, kTile))
        return cudaErrorInvalidValue;
    const bool pages = a.mode == kScorePages;
    if (a.H == 64)
        return pages ? launch_mq<64, 4, true>(map, a, groups_per_seq, n_groups, s)
                     : launch_mq<64, 4, false>(map, a, groups_per_seq, n_groups, s);
    if (a.H == 128)
        return pages ? launch_mq<128, 2, true>(map, a, groups_per_seq, n_groups, s)
                     : launch_mq<128, 2, false>(map, a, groups_per_seq, n_groups, s);
    return cudaErrorInvalidValue;
}

}  // namespace lsa
