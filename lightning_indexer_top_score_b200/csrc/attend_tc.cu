// attend_tc.cu -- Hybrid Sparse Attention forward on the 5th-generation tensor cores, one query
// per pair of CTAs (a thread-block cluster of two).
//
// Paper: Sec. 2.2 (u_t = Attn over the MLA latent rows c_s of S_t), Sec. 3.1 (S_t = sink U swa U
// S_sparse; the fixed tokens take part in the same softmax, Fig. 1), Sec. 4.1.1 (HFA: the
// contiguous and gathered branches merged by online-softmax rescaling).
//
// The 128 heads are the MMA's M = 128 rows.  The 576 latent dims are split between the two CTAs
// of a cluster: rank 0 owns dims 0-255 and 512-575 (chunks 0-3 and 8 of 64 dims), rank 1 owns
// dims 256-511 (chunks 4-7).  Each rank
//   - keeps its part of Q in TMEM and uses it as the MMA's A operand (no shared-memory re-reads
//     of Q per MMA),
//   - gathers only its chunks of each key row (16-byte cp.async by seven producer warps; a
//     TMA tile::gather4 moves only 512 bytes per instruction and its issue rate capped the
//     gather near 12 GB/s per SM) -- every latent row crosses HBM once for the pair,
//   - computes the partial S = Q_part K_part^T of a 64-key tile (N = 64: an MMA of N = 64
//     costs about what one of N = 32 does, and each tile's exchange and barrier latencies are
//     paid once per 64 keys),
//   - sends its partial S to the twin through distributed shared memory (st.async stores that
//     complete the twin's barrier by byte count) and adds the twin's, so both hold the same
//     full S (fp32 addition is commutative) and the same softmax,
//   - accumulates O += P V for its own 256 value dims (its chunks 0-3 are exactly those dims),
//     with P in TMEM as the A operand and V read MN-major from the gathered tile.
// O is rescaled lazily: only when a head's running max grows by more than 2^8 is O read back and
// scaled; otherwise P is formed against the stale max, which is exact.
//
// TMEM (512 columns): Q part [0,160) | S [160,224) | P (bf16 pairs) [224,256) | O [256,512); S
// and P hold one tile each.
// Warp roles (384 threads): warps 0-3 load Q_part, then softmax + exchange + epilogue (thread =
// head = TMEM lane), warps 4-10 producers (gathers into a ring of 3 stages of 64 keys; key
// positions are resolved and validated at set-up into shared memory), warp 11 TMEM allocator +
// single-thread MMA issuer.
// Every pipeline wait is bounded (LSA_DEVERR_TIMEOUT); the two cluster barriers (after set-up,
// before exit) are reached by both CTAs unconditionally.
//
// Grid: (query rows, 2 ranks, key splits) with clusters of (1, 2, 1); key splits are merged by
// hfa_combine_kernel.
#include <cstring>
#include <type_traits>

#include "lsa_internal.cuh"
#include "score_tc.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace tc;

constexpr int DQK = 576;
constexpr int NK = 64;       // keys per tile
constexpr int STAGES = 3;
constexpr int HEADS = 128;
constexpr int DVH = 256;     // value dims per rank
constexpr int kProducerWarps = 7;
constexpr int kMmaWarp = 4 + kProducerWarps;
constexpr int kThreads = 32 * (kMmaWarp + 1);
constexpr int kMaxOwn = 5;   // chunks of rank 0 (rank 1 owns 4)
constexpr float kRescaleLog2 = 8.f;

constexpr int kChunkBytes = NK * 128;              // 8192
constexpr int kStageBytes = kMaxOwn * kChunkBytes; // 40960
constexpr int kXBytes = HEADS * NK * 4;            // 32768: one partial-S exchange buffer
constexpr int OFF_KV = 0;
constexpr int OFF_X = OFF_KV + STAGES * kStageBytes;
constexpr int OFF_OK = OFF_X + 2 * kXBytes;
constexpr int OFF_BAR = OFF_OK + 64;
constexpr int kNumBars = 2 * STAGES + 8;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kPosTiles = 32;                      // tiles whose positions are staged at set-up
constexpr int OFF_POS = OFF_MISC + 16;
constexpr int OFF_IDX = OFF_POS + kPosTiles * NK * 4;  // the row's gathered indices
constexpr int kSmem = OFF_IDX + kMaxSelect * 4;
constexpr int kSmemLaunch = kSmem + 1024;          // slack to align the base to 1024
static_assert(kSmemLaunch <= 232448, "shared memory plan exceeds 227 KB");

constexpr uint32_t TQ = 0, TS = 160, TP = 224, TO = 256;

__device__ __forceinline__ int own_chunks(uint32_t rank) { return rank == 0 ? 5 : 4; }
__device__ __forceinline__ int own_chunk(uint32_t rank, int cl) {
    return rank == 0 ? (cl < 4 ? cl : 8) : 4 + cl;
}

struct RowKeys {
    int64_t n_sink, n_swa, swa_lo, n_sp, dyn_lo, dyn_hi;
    const int32_t *idx;
};

// Position of virtual key v (sink | window | gathered), -1 if none or invalid.
__device__ __forceinline__ int64_t key_pos(const RowKeys &L, int64_t v, int32_t *err) {
    if (v < L.n_sink) return v;
    v -= L.n_sink;
    if (v < L.n_swa) return L.swa_lo + v;
    v -= L.n_swa;
    if (v >= L.n_sp) return -1;
    const int64_t p = L.idx[v];
    if (p >= L.dyn_lo && p < L.dyn_hi && (v == 0 || L.idx[v - 1] < p)) return p;
    raise_error(err, LSA_DEVERR_INDEX);
    return -1;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kThreads, 1) hfa_tc_kernel(const __grid_constant__ CUtensorMap cmap,
                                                        AttendArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    uint8_t *kv_s = sm + OFF_KV;
    float *xbuf = reinterpret_cast<float *>(sm + OFF_X);  // [2][NK/4][HEADS][4]
    uint64_t *tile_mask = reinterpret_cast<uint64_t *>(sm + OFF_OK);  // bit j: key j valid
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *empty = full + STAGES;
    uint64_t *sfull = empty + STAGES;  // S of the tile written
    uint64_t *sfree = sfull + 1;       // the softmax has read S of the tile
    uint64_t *pfull = sfree + 1;       // P of the tile written
    uint64_t *pvdone = pfull + 1;      // O += P V of the tile completed
    // completed by the twin's st.async bytes: its partial S of the tile is in my xbuf.  No
    // "buffer free" signal is needed: I write the twin's buffer bb for tile i + 2 only after its
    // tile i + 1 data reached me, which it sent after reading its buffer bb for tile i.
    uint64_t *xfull = pvdone + 1;
    uint64_t *drain = xfull + 2;
    uint64_t *qready = drain + 1;  // Q_part is in TMEM (the softmax warps' 128 arrivals)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    int *nsp_s = reinterpret_cast<int *>(sm + OFF_MISC + 8);
    int32_t *pos_s = reinterpret_cast<int32_t *>(sm + OFF_POS);  // [kPosTiles][NK]
    int32_t *idx_s = reinterpret_cast<int32_t *>(sm + OFF_IDX);  // [K]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t twin = rank ^ 1u;
    const int nc = own_chunks(rank);
    const int64_t r = blockIdx.x;
    const int split = blockIdx.z;
    const int64_t b = r / a.T;
    const int64_t t = a.q_pos[r];
    const int64_t len = a.kv_len[b];
    // (both CTAs of a cluster take every early exit below together: same row, same split)
    if (!(t >= 0 && t < len && len <= a.L_max)) {
        if (tid == 0 && rank == 0 && split == 0) raise_error(a.err, LSA_DEVERR_QPOS);
        return;
    }
    if (tid < HEADS) {
        // start this head's Q_part on its way to L2 now; it is read into TMEM after set-up
        const char *qrow = reinterpret_cast<const char *>(a.q + (r * a.H + tid) * (int64_t)DQK);
        for (int cl = 0; cl < nc; ++cl)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(qrow + own_chunk(rank, cl) * 128));
    }
    const Regions g = regions_of(t, a.Ks, a.Kw);
    RowKeys L;
    L.n_sink = g.sink_hi;
    L.n_swa = g.swa_hi - g.swa_lo;
    L.swa_lo = g.swa_lo;
    L.dyn_lo = g.dyn_lo;
    L.dyn_hi = g.dyn_hi;
    {
        // the first two tiles of this split, where they fall in the sink or the window (their
        // positions need no index list), start on their way to L2 before the set-up below
        const int ns0 = a.n_split;
        if (tid < 2 * NK) {
            const int64_t v = ((int64_t)split + (int64_t)(tid / NK) * ns0) * NK + tid % NK;
            int64_t p = -1;
            if (v < L.n_sink)
                p = v;
            else if (v < L.n_sink + L.n_swa)
                p = L.swa_lo + (v - L.n_sink);
            if (p >= 0) {
                const char *row = reinterpret_cast<const char *>(a.c + (b * a.L_max + p) * DQK);
                for (int cl = 0; cl < nc; ++cl)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(row + own_chunk(rank, cl) * 128));
            }
        }
    }
    // ---- set-up.  The barriers are made first; the row's gathered indices are read once
    // (coalesced) into shared memory and counted; the key positions of the split are resolved
    // from there.  Then the producers start at once, while the softmax warps load Q_part into
    // TMEM (the MMA issuers wait for it) and only the softmax waits for the twin's barriers.
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 32 * kProducerWarps + 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(sfull, 1);
        mbar_init(sfree, 128);
        mbar_init(pfull, 128);
        mbar_init(pvdone, 1);
        mbar_init(&xfull[0], 1);
        mbar_init(&xfull[1], 1);
        mbar_init(drain, 1);
        mbar_init(qready, 128);
        *abort = 0;
        *nsp_s = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    {
        const int32_t *gidx = a.idx + r * a.K;
        int c = 0;
        for (int i = tid; i < a.K; i += kThreads) {
            const int32_t v = gidx[i];
            idx_s[i] = v;
            c += (v >= 0);
        }
        if (c) atomicAdd(nsp_s, c);
    }
    __syncthreads();
    L.idx = idx_s;
    L.n_sp = *nsp_s;
    const int64_t n_total = L.n_sink + L.n_swa + L.n_sp;
    const int64_t ntiles = (n_total + NK - 1) / NK;
    // split s takes tiles s, s + ns, s + 2 ns, ...: every split gets its share of the window's
    // contiguous tiles and of the gathered ones
    const int ns = a.n_split;
    const int n = (int)(split < ntiles ? (ntiles - split + ns - 1) / ns : 0);
    auto vkey = [&](int i, int j) -> int64_t { return ((int64_t)split + (int64_t)i * ns) * NK + j; };
    const int H = a.H;  // == 128
    if (n == 0) {
        // an empty split: a zero partial with lse = -inf (only reachable with several splits)
        if (a.n_split > 1) {
            for (int i = tid; i < HEADS * DVH; i += kThreads) {
                const int h = i / DVH, d = i - h * DVH;
                a.part_o[((r * H + h) * a.n_split + split) * (int64_t)512 + rank * DVH + d] = 0.f;
            }
            if (rank == 0)
                for (int h = tid; h < HEADS; h += kThreads)
                    a.part_lse[(r * H + h) * a.n_split + split] = -INFINITY;
        }
        return;
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    {
        // positions of the first kPosTiles tiles of this split (all threads); the producers
        // read them from shared memory
        const int np = (n < kPosTiles ? n : kPosTiles) * NK;
        for (int e = tid; e < np; e += kThreads)
            pos_s[e] = (int32_t)key_pos(L, vkey(e / NK, e % NK), a.err);
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;
    cluster_arrive();  // my barriers exist; the twin waits for this before its first remote arrive

    if (warp >= 4 && warp < kMmaWarp) {
        // ------------------------------------------------------------ producers
        // Each thread copies 16-byte pieces of this rank's chunks of the tile's key rows with
        // cp.async (zero-filled for an empty slot), swizzled in place to the SWIZZLE_128B K-major
        // layout, then lets the stage barrier count its arrival once those copies have landed
        // (cp.async.mbarrier.arrive.noinc): no producer thread waits for its own copies, so up
        // to STAGES tiles are in flight.  Lane 0 of the first producer warp also publishes the
        // tile's validity mask with a plain arrival.
        const int ptid = tid - 128;
        const int per_row = nc * 8;  // 16-byte pieces of this rank per key row
        constexpr int kStep = 32 * kProducerWarps;
        const int dj = kStep / per_row, drem = kStep - dj * per_row;
        const int j0 = ptid / per_row, rem0 = ptid - j0 * per_row;
        const __nv_bfloat16 *cseq = a.c + b * a.L_max * DQK;
        int tma_issued = 0;  // tiles up to which this thread issued TMA boxes
        for (int i = 0; i < n; ++i) {
            const int s = i % STAGES;
            // one lane per warp polls the stage barrier (256 polling threads would compete
            // with the tensor core for the shared-memory port)
            bool ok = true;
            if (i >= STAGES && lane == 0)
                ok = mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, abort, a.err);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            __syncwarp();
            if (!ok) break;
            // positions come from shared memory for the staged tiles; past them each thread
            // resolves the rows it copies
            const bool staged = i < kPosTiles;
            const int64_t p0 = staged ? (int64_t)pos_s[i * NK + lane] : key_pos(L, vkey(i, lane), a.err);
            const int64_t p1 =
                staged ? (int64_t)pos_s[i * NK + 32 + lane] : key_pos(L, vkey(i, 32 + lane), a.err);
            // a tile of 64 consecutive valid positions (the window) is one 2-D TMA box per
            // chunk, issued by one thread; the others are gathered row by row
            const int64_t first = __shfl_sync(0xFFFFFFFFu, p0, 0);
            const bool contig = __all_sync(0xFFFFFFFFu, first >= 0 && p0 == first + lane &&
                                                            p1 == first + 32 + lane);
            uint8_t *base = kv_s + s * kStageBytes;
            if (!contig) {
                int j = j0, rem = rem0;
                for (int k = ptid; k < NK * per_row; k += kStep) {
                    const int cl = rem >> 3, pc = rem & 7;
                    const int64_t pos = staged ? (int64_t)pos_s[i * NK + j] : key_pos(L, vkey(i, j), a.err);
                    cp_async16(base + cl * kChunkBytes + j * 128 + ((pc ^ (j & 7)) << 4),
                               pos >= 0 ? cseq + pos * DQK + own_chunk(rank, cl) * 64 + pc * 8 : cseq,
                               pos >= 0 ? 16 : 0);
                    j += dj;
                    rem += drem;
                    if (rem >= per_row) {
                        rem -= per_row;
                        ++j;
                    }
                }
            }
            cp_async_arrive_noinc(&full[s]);
            if (warp == 4) {
                const uint64_t vmask = ((uint64_t)__ballot_sync(0xFFFFFFFFu, p1 >= 0) << 32) |
                                       __ballot_sync(0xFFFFFFFFu, p0 >= 0);
                if (lane == 0) {
                    tile_mask[s] = vmask;
                    // the mask's arrival; for a TMA tile it also expects the boxes' bytes
                    mbar_expect_tx(&full[s], contig ? (uint32_t)(nc * kChunkBytes) : 0u);
                    if (contig) {
                        const int row = (int)(b * a.L_max + first);
                        for (int cl = 0; cl < nc; ++cl)
                            tma_load_2d(base + cl * kChunkBytes, &cmap, own_chunk(rank, cl) * 64,
                                        row, &full[s]);
                        tma_issued = i + 1;
                    }
                }
            }
        }
        cp_async_wait_all();  // nothing of this thread is in flight when the CTA leaves
        if (warp == 4 && lane == 0 && *abort) {
            // error path: let the TMA boxes already issued land (bounded) before leaving
            for (int k = tma_issued > STAGES ? tma_issued - STAGES : 0; k < tma_issued; ++k) {
                const uint64_t ts = globaltimer();
                while (!mbar_try(&full[k % STAGES], (k / STAGES) & 1))
                    if (globaltimer() - ts > 100000000ull) break;
            }
        }
        cluster_wait();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        // A tcgen05.mma of M = 128, K = 16 costs about the same to issue for any N up to 128,
        // so S = Q_part K_part^T is one chain of N = 64 (keys) MMAs per tile; then O += P V.
        if (lane == 0) {
            const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) |
                                     ((uint32_t)(NK >> 3) << 17) | ((uint32_t)(HEADS >> 4) << 24);
            const uint32_t idesc_pv = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(DVH >> 3) << 17) |
                                      ((uint32_t)(HEADS >> 4) << 24);
            const uint32_t kv_addr = smem_u32(kv_s);
            // the k-steps are a compile-time count (20 for rank 0, 16 for rank 1): the chain is
            // unrolled over descriptors built once for stage 0 and shifted per stage (the
            // start-address field holds every shared-memory address without carry)
            auto run = [&](auto ks_c) {
                constexpr int KS = decltype(ks_c)::value;
                if (!mbar_wait(qready, 0, abort, a.err)) return;  // Q_part is in TMEM
                fence_after();
                uint64_t dk[KS];
#pragma unroll
                for (int k = 0; k < KS; ++k)
                    dk[k] = smem_desc(kv_addr + (k >> 2) * kChunkBytes + (k & 3) * 32, 16, 1024, 2);
                auto issue_s = [&](int i) -> bool {
                    const int s = i % STAGES;
                    if (!mbar_wait(&full[s], (i / STAGES) & 1, abort, a.err)) return false;
                    // S holds one tile at a time: the softmax must have read tile i - 1
                    if (i >= 1 && !mbar_wait(sfree, (i - 1) & 1, abort, a.err)) return false;
                    fence_proxy_async();  // the cp.async writes of the stage, seen by the MMA
                    fence_after();
                    const uint64_t soff = (uint64_t)((s * kStageBytes) >> 4);
#pragma unroll
                    for (int k = 0; k < KS; ++k)
                        umma_bf16_ts(tmem + TS, tmem + TQ + k * 8, dk[k] + soff, idesc_s, k > 0);
                    umma_commit(sfull);
                    return true;
                };
                bool live = issue_s(0);
                for (int i = 0; i < n && live; ++i) {
                    if (i + 1 < n && !issue_s(i + 1)) break;
                    const int s = i % STAGES;
                    if (!mbar_wait(pfull, i & 1, abort, a.err)) break;
                    fence_after();
#pragma unroll
                    for (int ks = 0; ks < NK / 16; ++ks) {
                        const uint64_t bd = smem_desc(kv_addr + s * kStageBytes + ks * 2048,
                                                      kChunkBytes, 1024, 2);
                        umma_bf16_ts(tmem + TO, tmem + TP + ks * 8, bd, idesc_pv,
                                     (i > 0 || ks > 0) ? 1u : 0u);
                    }
                    // the stage is free once this P V has read it (S of the tile completed
                    // before the softmax produced P)
                    umma_commit(&empty[s]);
                    umma_commit(pvdone);
                }
            };
            if (nc == 5)
                run(std::integral_constant<int, 20>());
            else
                run(std::integral_constant<int, 16>());
            umma_commit(drain);
            const uint64_t ts = globaltimer();
            while (!mbar_try(drain, 0))
                if (globaltimer() - ts > kWaitNs) {
                    raise_error(a.err, LSA_DEVERR_TIMEOUT);
                    break;
                }
        }
        cluster_wait();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int h = tid;  // head = TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        {
            // Q_part into TMEM: thread h writes row h, local chunk cl to columns
            // [32 cl, 32 cl + 32); the loads of three chunks are in flight per round
            const uint4 *qr = reinterpret_cast<const uint4 *>(a.q + (r * H + h) * (int64_t)DQK);
            for (int c0 = 0; c0 < nc; c0 += 3) {
                uint4 x[3][8];
#pragma unroll
                for (int u = 0; u < 3; ++u)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        x[u][k] = (c0 + u < nc) ? __ldg(qr + own_chunk(rank, c0 + u) * 8 + k)
                                                : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int u = 0; u < 3; ++u) {
                    if (c0 + u >= nc) break;
                    uint32_t v[32];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        v[4 * k] = x[u][k].x;
                        v[4 * k + 1] = x[u][k].y;
                        v[4 * k + 2] = x[u][k].z;
                        v[4 * k + 3] = x[u][k].w;
                    }
                    tmem_st32(tmem + lane_base + TQ + (c0 + u) * 32, v);
                }
            }
            tmem_wait_st();
            fence_before();
            mbar_arrive(qready);
        }
        cluster_wait();  // the twin's barriers exist before my first remote arrive
        const uint32_t o_tmem = tmem + lane_base + TO;
        const uint32_t x_twin = mapa(xbuf, twin);  // the twin's exchange buffers
        const uint32_t xfull_twin[2] = {mapa(&xfull[0], twin), mapa(&xfull[1], twin)};
        float m_ref = -INFINITY, l = 0.f;
        bool nonfinite = false, live = true;
        for (int i = 0; i < n; ++i) {
            const int bb = i & 1, s = i % STAGES;
            bool ok = mbar_wait(sfull, i & 1, abort, a.err);
            ok = ok && mbar_wait(&full[s], (i / STAGES) & 1, abort, a.err);
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                live = false;
                break;
            }
            fence_after();
            uint32_t v[NK];
            tmem_ld64(tmem + lane_base + TS, v);
            tmem_wait_ld();
            fence_before();
            mbar_arrive(sfree);
            // this tile's twin data (32 KB) completes my barrier xfull[bb]
            if (tid == 0) mbar_expect_tx(&xfull[bb], kXBytes);
            // send my partial S row to the twin (layout [NK/4][HEADS][4] floats per buffer)
#pragma unroll
            for (int k = 0; k < NK / 4; ++k)
                st_async_v4(x_twin + bb * kXBytes + (k * HEADS + h) * 16,
                            make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]),
                            xfull_twin[bb]);
            // add the twin's partial S row in place (v holds the unscaled logits afterwards; an
            // empty slot gets -inf); scale_log2 > 0 is applied once to the max and folded into
            // the exponent below
            const bool okx = mbar_wait_cluster(&xfull[bb], (i >> 1) & 1, abort, a.err);
            if (!__all_sync(0xFFFFFFFFu, okx)) {
                live = false;
                break;
            }
            const uint64_t vmask = tile_mask[s];
            const float *xrow = xbuf + bb * (NK / 4) * HEADS * 4 + h * 4;
            if (vmask == ~0ull) {
#pragma unroll
                for (int k = 0; k < NK / 4; ++k) {
                    const float4 x = *reinterpret_cast<const float4 *>(xrow + k * HEADS * 4);
                    v[4 * k] = __float_as_uint(__uint_as_float(v[4 * k]) + x.x);
                    v[4 * k + 1] = __float_as_uint(__uint_as_float(v[4 * k + 1]) + x.y);
                    v[4 * k + 2] = __float_as_uint(__uint_as_float(v[4 * k + 2]) + x.z);
                    v[4 * k + 3] = __float_as_uint(__uint_as_float(v[4 * k + 3]) + x.w);
                }
            } else {
#pragma unroll
                for (int k = 0; k < NK / 4; ++k) {
                    const float4 x = *reinterpret_cast<const float4 *>(xrow + k * HEADS * 4);
                    const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 4 * k + e;
                        v[j] = __float_as_uint(((vmask >> j) & 1u) ? __uint_as_float(v[j]) + xs[e]
                                                                   : -INFINITY);
                    }
                }
            }
            float mt;
            {  // pairwise max tree
                float m16[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    m16[j] = fmaxf(fmaxf(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1])),
                                   fmaxf(__uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
#pragma unroll
                for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                    for (int j = 0; j < w; ++j) m16[j] = fmaxf(m16[j], m16[j + w]);
                mt = m16[0] * a.scale_log2;  // -inf stays -inf
            }
            const bool need = (m_ref == -INFINITY) ? (mt > -INFINITY) : (mt > m_ref + kRescaleLog2);
            if (__any_sync(0xFFFFFFFFu, need)) {
                float alpha = 1.f, m_new = m_ref;
                if (need) {
                    m_new = fmaxf(m_ref, mt);
                    alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - m_new);
                }
                if (i > 0) {
                    // O holds the P V of tiles < i: wait for the last one, then scale in place
                    const bool okp = mbar_wait(pvdone, (i - 1) & 1, abort, a.err);
                    if (!__all_sync(0xFFFFFFFFu, okp)) {
                        live = false;
                        break;
                    }
                    fence_after();
#pragma unroll 1
                    for (int ch = 0; ch < DVH / 32; ++ch) {
                        uint32_t ov[32];
                        tmem_ld32(o_tmem + ch * 32, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
                        tmem_st32(o_tmem + ch * 32, ov);
                    }
                    tmem_wait_st();
                    fence_before();
                }
                l *= alpha;
                m_ref = m_new;
            }
            uint32_t pk[NK / 2];
            float rs0 = 0.f, rs1 = 0.f;
            const float mref = (m_ref == -INFINITY) ? 0.f : m_ref;  // all p = 0 then (z = -inf)
            const float sc = a.scale_log2;
#pragma unroll
            for (int j = 0; j < NK; j += 2) {
                const float p0 = fast_exp2(fmaf(__uint_as_float(v[j]), sc, -mref));
                const float p1 = fast_exp2(fmaf(__uint_as_float(v[j + 1]), sc, -mref));
                rs0 += p0;
                rs1 += p1;
                pk[j >> 1] = pack_bf16(p0, p1);
            }
            const float rs = rs0 + rs1;
            nonfinite |= !isfinite(rs);  // a NaN or infinite logit always reaches the row sum
            l += rs;
            if (i >= 1) {
                // P holds one tile: the P V of tile i - 1 must have completed
                const bool okp = mbar_wait(pvdone, (i - 1) & 1, abort, a.err);
                if (!__all_sync(0xFFFFFFFFu, okp)) {
                    live = false;
                    break;
                }
            }
            tmem_st32(tmem + lane_base + TP, pk);
            tmem_wait_st();
            fence_before();
            mbar_arrive(pfull);
        }
        if (nonfinite) raise_error(a.err, LSA_DEVERR_NONFINITE);
        bool okf = live && mbar_wait(pvdone, (n - 1) & 1, abort, a.err);
        if (__all_sync(0xFFFFFFFFu, okf)) {
            fence_after();
            // the key ring is idle now (every MMA that read it has completed): O goes out through
            // it, so that each store instruction writes one head's contiguous 512 bytes instead
            // of 16 bytes of 32 different heads.  A warp stages and copies out only its own 32
            // head rows (its TMEM lanes), so __syncwarp orders the two phases.
            fence_proxy_async();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const float lse = l > 0.f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
            constexpr int kStgRow = 528;  // bytes per staged row: 512 + 16 (spreads the banks)
            uint8_t *stg = kv_s;
            const int h0 = warp * 32;
            // O row h, 32 columns at a time; the TMEM load of the next 32 columns is in flight
            // while these are scaled and staged
            uint32_t ov[2][32];
            if (a.n_split == 1) {
                // bf16 output: the whole 256-dim row (512 bytes) staged at once
                tmem_ld32(o_tmem, ov[0]);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < DVH / 32; ++ch) {
                    if (ch + 1 < DVH / 32) tmem_ld32(o_tmem + (ch + 1) * 32, ov[(ch + 1) & 1]);
                    const uint32_t *w = ov[ch & 1];
#pragma unroll
                    for (int j = 0; j < 32; j += 8)
                        *reinterpret_cast<uint4 *>(stg + h * kStgRow + ch * 64 + j * 2) = make_uint4(
                            pack_bf16(__uint_as_float(w[j]) * inv, __uint_as_float(w[j + 1]) * inv),
                            pack_bf16(__uint_as_float(w[j + 2]) * inv, __uint_as_float(w[j + 3]) * inv),
                            pack_bf16(__uint_as_float(w[j + 4]) * inv, __uint_as_float(w[j + 5]) * inv),
                            pack_bf16(__uint_as_float(w[j + 6]) * inv, __uint_as_float(w[j + 7]) * inv));
                    tmem_wait_ld();
                }
                __syncwarp();
#pragma unroll 4
                for (int i = 0; i < 32; ++i) {
                    const int hr = h0 + i;
                    const uint4 v = *reinterpret_cast<const uint4 *>(stg + hr * kStgRow + lane * 16);
                    *reinterpret_cast<uint4 *>(a.out + (r * H + hr) * (int64_t)512 + rank * DVH +
                                               lane * 8) = v;
                }
            } else {
                // fp32 partial output: two halves of 128 dims (512 bytes per head each)
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(o_tmem + half * 128, ov[0]);
                    tmem_wait_ld();
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        if (ch + 1 < 4) tmem_ld32(o_tmem + half * 128 + (ch + 1) * 32, ov[(ch + 1) & 1]);
                        const uint32_t *w = ov[ch & 1];
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4 *>(stg + h * kStgRow + ch * 128 + j * 4) =
                                make_float4(__uint_as_float(w[j]) * inv,
                                            __uint_as_float(w[j + 1]) * inv,
                                            __uint_as_float(w[j + 2]) * inv,
                                            __uint_as_float(w[j + 3]) * inv);
                        tmem_wait_ld();
                    }
                    __syncwarp();
#pragma unroll 4
                    for (int i = 0; i < 32; ++i) {
                        const int hr = h0 + i;
                        const float4 v =
                            *reinterpret_cast<const float4 *>(stg + hr * kStgRow + lane * 16);
                        *reinterpret_cast<float4 *>(
                            a.part_o + ((r * H + hr) * a.n_split + split) * (int64_t)512 +
                            rank * DVH + half * 128 + lane * 4) = v;
                    }
                    __syncwarp();  // the staged rows are rewritten by the next half
                }
            }
            if (rank == 0) {
                if (a.n_split == 1)
                    a.lse[r * H + h] = lse;
                else
                    a.part_lse[(r * H + h) * a.n_split + split] = lse;
            }
        }
    }

    // ---- tear-down: free TMEM, then leave together (the twin may still arrive on my barriers)
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == kMmaWarp) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
    __syncwarp();
    cluster_sync();
}

}  // namespace

int attend_tc_tile() { return NK; }

cudaError_t launch_attend_tc(const AttendArgs &a, int64_t rows, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    if (rows > 0x7FFFFFFF) return cudaErrorInvalidValue;
    if (a.L_max > 0x7FFFFFFFll) return cudaErrorInvalidValue;  // positions are staged as int32
    const int64_t nb = rows / a.T;  // sequences
    if (nb * a.L_max >= 0x7FFFFFFFll) return cudaErrorInvalidValue;  // TMA row coordinate
    // latent rows as a 2-D tensor [nb * L_max, 576] bf16, boxes of 64 dims x NK rows (SWIZZLE_128B)
    CUtensorMap cmap;
    if (!make_tmap_2d_bf16(&cmap, a.c, DQK, (uint64_t)(nb * a.L_max), 64, NK))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(hfa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemLaunch);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)rows, 2u, (unsigned)a.n_split);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemLaunch;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 2;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, hfa_tc_kernel, cmap, a);
    if (e != cudaSuccess) return e;
    return launched();
}

}  // namespace lsa
