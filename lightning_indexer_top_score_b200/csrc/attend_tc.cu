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
//   - gathers only its chunks of each key row (16-byte cp.async by eight producer warps; a
//     TMA tile::gather4 moves only 512 bytes per instruction and its issue rate capped the
//     gather near 12 GB/s per SM) -- every latent row crosses HBM once for the pair,
//   - computes the partial S = Q_part K_part^T of a 32-key tile (N = 32),
//   - sends its partial S to the twin through distributed shared memory (st.async stores that
//     complete the twin's barrier by byte count) and adds the twin's, so both hold the same
//     full S (fp32 addition is commutative) and the same softmax,
//   - accumulates O += P V for its own 256 value dims (its chunks 0-3 are exactly those dims),
//     with P in TMEM as the A operand and V read MN-major from the gathered tile.
// O is rescaled lazily: only when a head's running max grows by more than 2^8 is O read back and
// scaled; otherwise P is formed against the stale max, which is exact.
//
// TMEM (512 columns): Q part [0,160) | S_A [160,192) | S_B [192,224) | P x2 (bf16 pairs)
// [224,256) | O [256,512).
// Warp roles (448 threads): warps 0-3 softmax + exchange + epilogue (thread = head = TMEM lane),
// warps 4-11 producers (gathers into a ring of 6 stages; key positions are resolved and validated
// at set-up into shared memory), warp 12 TMEM allocator + MMA issuer A, warp 13 MMA issuer B.
// Every pipeline wait is bounded (LSA_DEVERR_TIMEOUT); the two cluster barriers (after set-up,
// before exit) are reached by both CTAs unconditionally.
//
// Grid: (query rows, 2 ranks, key splits) with clusters of (1, 2, 1); key splits are merged by
// hfa_combine_kernel.
#include <cstring>
#include <type_traits>

#include "lsa_internal.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace tc;

constexpr int DQK = 576;
constexpr int NK = 32;       // keys per tile
constexpr int STAGES = 6;
constexpr int HEADS = 128;
constexpr int DVH = 256;     // value dims per rank
constexpr int kProducerWarps = 8;
constexpr int kMmaWarp = 4 + kProducerWarps;
constexpr int kThreads = 32 * (kMmaWarp + 2);  // + MMA issuer B
constexpr int kMaxOwn = 5;   // chunks of rank 0 (rank 1 owns 4)
constexpr float kRescaleLog2 = 8.f;

constexpr int kChunkBytes = NK * 128;              // 4096
constexpr int kStageBytes = kMaxOwn * kChunkBytes; // 20480
constexpr int kXBytes = HEADS * NK * 4;            // 16384: one partial-S exchange buffer
constexpr int OFF_KV = 0;
constexpr int OFF_X = OFF_KV + STAGES * kStageBytes;
constexpr int OFF_OK = OFF_X + 2 * kXBytes;
constexpr int OFF_BAR = OFF_OK + 64;
constexpr int kNumBars = 2 * STAGES + 2 + 2 * 4;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kPosTiles = 64;                      // tiles whose positions are staged at set-up
constexpr int OFF_POS = OFF_MISC + 16;
constexpr int kSmem = OFF_POS + kPosTiles * NK * 4;
constexpr int kSmemLaunch = kSmem + 1024;          // slack to align the base to 1024
static_assert(kSmemLaunch <= 232448, "shared memory plan exceeds 227 KB");

constexpr uint32_t TQ = 0, TSA = 160, TSB = 192, TP0 = 224, TO = 256;

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

__global__ void __launch_bounds__(kThreads, 1) hfa_tc_kernel(AttendArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    uint8_t *kv_s = sm + OFF_KV;
    float *xbuf = reinterpret_cast<float *>(sm + OFF_X);  // [2][NK/4][HEADS][4]
    uint32_t *tile_mask = reinterpret_cast<uint32_t *>(sm + OFF_OK);  // bit j: key j valid
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *empty = full + STAGES;
    uint64_t *sfull = empty + STAGES;  // both halves of S of the tile written (2 commits)
    uint64_t *sfree = sfull + 1;       // the softmax has read S of the tile
    uint64_t *pfull = sfree + 1;
    uint64_t *pvdone = pfull + 2;
    // completed by the twin's st.async bytes: its partial S of the tile is in my xbuf.  No
    // "buffer free" signal is needed: I write the twin's buffer bb for tile i + 2 only after its
    // tile i + 1 data reached me, which it sent after reading its buffer bb for tile i.
    uint64_t *xfull = pvdone + 2;
    uint64_t *drain = xfull + 2;  // [2]: one per MMA issuer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    int *nsp_s = reinterpret_cast<int *>(sm + OFF_MISC + 8);
    int32_t *pos_s = reinterpret_cast<int32_t *>(sm + OFF_POS);  // [kPosTiles][NK]

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
    const Regions g = regions_of(t, a.Ks, a.Kw);
    RowKeys L;
    L.n_sink = g.sink_hi;
    L.n_swa = g.swa_hi - g.swa_lo;
    L.swa_lo = g.swa_lo;
    L.dyn_lo = g.dyn_lo;
    L.dyn_hi = g.dyn_hi;
    L.idx = a.idx + r * a.K;
    if (tid == 0) *nsp_s = 0;
    __syncthreads();
    {
        int c = 0;
        for (int i = tid; i < a.K; i += kThreads) c += (L.idx[i] >= 0);
        if (c) atomicAdd(nsp_s, c);
    }
    __syncthreads();
    L.n_sp = *nsp_s;
    const int64_t n_total = L.n_sink + L.n_swa + L.n_sp;
    const int64_t ntiles = (n_total + NK - 1) / NK;
    const int64_t t0 = (int64_t)split * a.tiles_per_split;
    int64_t t1 = t0 + a.tiles_per_split;
    if (t1 > ntiles) t1 = ntiles;
    const int n = (int)(t1 > t0 ? t1 - t0 : 0);
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

    // ---- set-up: barriers, TMEM, this rank's part of Q into TMEM, then meet the twin
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 32 * kProducerWarps + 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(sfull, 2);
        mbar_init(sfree, 128);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&pfull[s], 128);
            mbar_init(&pvdone[s], 1);
            mbar_init(&xfull[s], 1);
            mbar_init(&drain[s], 1);
        }
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp < 4) {
        // thread h writes row h of Q_part: chunk cl -> TMEM columns [32 cl, 32 cl + 32)
        const uint4 *qr = reinterpret_cast<const uint4 *>(a.q + (r * H + tid) * (int64_t)DQK);
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        for (int cl = 0; cl < nc; ++cl) {
            const int c = own_chunk(rank, cl);
            uint32_t v[32];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint4 x = __ldg(qr + c * 8 + k);
                v[4 * k] = x.x;
                v[4 * k + 1] = x.y;
                v[4 * k + 2] = x.z;
                v[4 * k + 3] = x.w;
            }
            tmem_st32(tmem + lane_base + TQ + cl * 32, v);
        }
        tmem_wait_st();
    }
    {
        // positions of the first kPosTiles tiles of this split (coalesced index reads, all
        // threads); the producer reads them from shared memory
        const int np = (n < kPosTiles ? n : kPosTiles) * NK;
        for (int e = tid; e < np; e += kThreads)
            pos_s[e] = (int32_t)key_pos(L, t0 * NK + e, a.err);
    }
    fence_before();
    __syncthreads();
    __syncwarp();
    cluster_sync();  // the twin's barriers exist before anyone arrives on them remotely
    fence_after();

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
        for (int i = 0; i < n; ++i) {
            const int s = i % STAGES;
            bool ok = true;
            if (i >= STAGES) ok = mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, abort, a.err);
            if (!__all_sync(0xFFFFFFFFu, ok)) break;
            // positions come from shared memory for the staged tiles; past them each thread
            // resolves the rows it copies
            const bool staged = i < kPosTiles;
            uint32_t vmask = 0;
            if (warp == 4) {
                const int64_t pos = staged ? (int64_t)pos_s[i * NK + lane]
                                           : key_pos(L, (t0 + i) * NK + lane, a.err);
                vmask = __ballot_sync(0xFFFFFFFFu, pos >= 0);
            }
            uint8_t *base = kv_s + s * kStageBytes;
            int j = j0, rem = rem0;
            for (int k = ptid; k < NK * per_row; k += kStep) {
                const int cl = rem >> 3, pc = rem & 7;
                const int64_t pos = staged ? (int64_t)pos_s[i * NK + j]
                                           : key_pos(L, (t0 + i) * NK + j, a.err);
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
            cp_async_arrive_noinc(&full[s]);
            if (warp == 4 && lane == 0) {
                tile_mask[s] = vmask;
                mbar_arrive(&full[s]);
            }
        }
        cp_async_wait_all();  // nothing of this thread is in flight when the CTA leaves
    } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
        // ------------------------------------------------------------ MMA issuers
        // Small-N MMAs cost about the same to issue whatever N is, and issues from two threads
        // overlap, so the S = Q_part K_part^T chain of a tile is split between two threads by
        // k-steps (issuer A: the first half into S_A, issuer B: the rest into S_B); the softmax
        // adds the two halves.  Issuer A also issues O += P V.
        if (lane == 0) {
            const bool is_a = warp == kMmaWarp;
            const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) |
                                     ((uint32_t)(NK >> 3) << 17) | ((uint32_t)(HEADS >> 4) << 24);
            const uint32_t idesc_pv = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(DVH >> 3) << 17) |
                                      ((uint32_t)(HEADS >> 4) << 24);
            const uint32_t kv_addr = smem_u32(kv_s);
            const uint32_t d_s = tmem + (is_a ? TSA : TSB);
            // the issuer's k-steps are a compile-time count (10 for rank 0, 8 for rank 1): the
            // chain is unrolled over descriptors built once for stage 0 and shifted per stage
            // (the start-address field holds every shared-memory address without carry)
            auto run = [&](auto kh_c) {
                constexpr int KH = decltype(kh_c)::value;
                const int k0 = is_a ? 0 : KH;
                uint64_t dk[KH];
#pragma unroll
                for (int k = 0; k < KH; ++k)
                    dk[k] = smem_desc(kv_addr + ((k0 + k) >> 2) * kChunkBytes + ((k0 + k) & 3) * 32,
                                      16, 1024, 2);
                auto issue_s = [&](int i) -> bool {
                    const int s = i % STAGES;
                    if (!mbar_wait(&full[s], (i / STAGES) & 1, abort, a.err)) return false;
                    // S holds one tile at a time: the softmax must have read tile i - 1
                    if (i >= 1 && !mbar_wait(sfree, (i - 1) & 1, abort, a.err)) return false;
                    fence_proxy_async();  // the cp.async writes of the stage, seen by the MMA
                    fence_after();
                    const uint64_t soff = (uint64_t)((s * kStageBytes) >> 4);
#pragma unroll
                    for (int k = 0; k < KH; ++k)
                        umma_bf16_ts(d_s, tmem + TQ + (k0 + k) * 8, dk[k] + soff, idesc_s, k > 0);
                    umma_commit(sfull);
                    return true;
                };
                bool live = issue_s(0);
                for (int i = 0; i < n && live; ++i) {
                    if (i + 1 < n && !issue_s(i + 1)) break;
                    if (!is_a) continue;
                    const int bb = i & 1, s = i % STAGES;
                    if (!mbar_wait(&pfull[bb], (i >> 1) & 1, abort, a.err)) break;
                    fence_after();
#pragma unroll
                    for (int ks = 0; ks < NK / 16; ++ks) {
                        const uint64_t bd = smem_desc(kv_addr + s * kStageBytes + ks * 2048,
                                                      kChunkBytes, 1024, 2);
                        umma_bf16_ts(tmem + TO, tmem + TP0 + bb * 16 + ks * 8, bd, idesc_pv,
                                     (i > 0 || ks > 0) ? 1u : 0u);
                    }
                    // the stage is free once this P V has read it (S of the tile, both halves,
                    // completed before the softmax produced P)
                    umma_commit(&empty[s]);
                    umma_commit(&pvdone[bb]);
                }
            };
            if (nc == 5)
                run(std::integral_constant<int, 10>());
            else
                run(std::integral_constant<int, 8>());
            uint64_t *dr = &drain[is_a ? 0 : 1];
            umma_commit(dr);
            const uint64_t ts = globaltimer();
            while (!mbar_try(dr, 0))
                if (globaltimer() - ts > kWaitNs) {
                    raise_error(a.err, LSA_DEVERR_TIMEOUT);
                    break;
                }
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int h = tid;  // head = TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
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
            uint32_t v[NK], vb[NK];
            tmem_ld32(tmem + lane_base + TSA, v);
            tmem_ld32(tmem + lane_base + TSB, vb);
            tmem_wait_ld();
            fence_before();
            mbar_arrive(sfree);
#pragma unroll
            for (int j = 0; j < NK; ++j)
                v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(vb[j]));
            // this tile's twin data (16 KB) completes my barrier xfull[bb]
            if (tid == 0) mbar_expect_tx(&xfull[bb], kXBytes);
            // send my partial S row to the twin (layout [NK/4][HEADS][4] floats per buffer)
#pragma unroll
            for (int k = 0; k < NK / 4; ++k)
                st_async_v4(x_twin + bb * kXBytes + (k * HEADS + h) * 16,
                            make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]),
                            xfull_twin[bb]);
            // add the twin's partial S row
            const bool okx = mbar_wait_cluster(&xfull[bb], (i >> 1) & 1, abort, a.err);
            if (!__all_sync(0xFFFFFFFFu, okx)) {
                live = false;
                break;
            }
            float z[NK];
            const uint32_t vmask = tile_mask[s];
#pragma unroll
            for (int k = 0; k < NK / 4; ++k) {
                const float4 x = *reinterpret_cast<const float4 *>(
                    xbuf + (bb * (NK / 4) + k) * HEADS * 4 + h * 4);
                const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 4 * k + e;
                    z[j] = ((vmask >> j) & 1u) ? (__uint_as_float(v[j]) + xs[e]) * a.scale_log2
                                               : -INFINITY;
                }
            }
            float mt;
            {  // pairwise max tree
                float m8[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    m8[j] = fmaxf(fmaxf(z[4 * j], z[4 * j + 1]), fmaxf(z[4 * j + 2], z[4 * j + 3]));
                mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                           fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
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
                    const bool okp = mbar_wait(&pvdone[(i - 1) & 1], ((i - 1) >> 1) & 1, abort,
                                               a.err);
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
#pragma unroll
            for (int j = 0; j < NK; j += 2) {
                const float p0 = fast_exp2(z[j] - mref);
                const float p1 = fast_exp2(z[j + 1] - mref);
                rs0 += p0;
                rs1 += p1;
                pk[j >> 1] = pack_bf16(p0, p1);
            }
            const float rs = rs0 + rs1;
            nonfinite |= !isfinite(rs);  // a NaN or infinite logit always reaches the row sum
            l += rs;
            if (i >= 2) {
                // P buffer bb is free once the P V of tile i-2 has completed
                const bool okp = mbar_wait(&pvdone[bb], ((i - 2) >> 1) & 1, abort, a.err);
                if (!__all_sync(0xFFFFFFFFu, okp)) {
                    live = false;
                    break;
                }
            }
            tmem_st16(tmem + lane_base + TP0 + bb * 16, pk);
            tmem_wait_st();
            fence_before();
            mbar_arrive(&pfull[bb]);
        }
        if (nonfinite) raise_error(a.err, LSA_DEVERR_NONFINITE);
        bool okf = live && mbar_wait(&pvdone[(n - 1) & 1], ((n - 1) >> 1) & 1, abort, a.err);
        if (__all_sync(0xFFFFFFFFu, okf)) {
            fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const float lse = l > 0.f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
#pragma unroll 1
            for (int ch = 0; ch < DVH / 32; ++ch) {
                uint32_t ov[32];
                tmem_ld32(o_tmem + ch * 32, ov);
                tmem_wait_ld();
                if (a.n_split == 1) {
                    __nv_bfloat16 *o = a.out + (r * H + h) * (int64_t)512 + rank * DVH + ch * 32;
#pragma unroll
                    for (int j = 0; j < 32; j += 8)
                        *reinterpret_cast<uint4 *>(o + j) = make_uint4(
                            pack_bf16(__uint_as_float(ov[j]) * inv, __uint_as_float(ov[j + 1]) * inv),
                            pack_bf16(__uint_as_float(ov[j + 2]) * inv, __uint_as_float(ov[j + 3]) * inv),
                            pack_bf16(__uint_as_float(ov[j + 4]) * inv, __uint_as_float(ov[j + 5]) * inv),
                            pack_bf16(__uint_as_float(ov[j + 6]) * inv, __uint_as_float(ov[j + 7]) * inv));
                } else {
                    float *o = a.part_o + ((r * H + h) * a.n_split + split) * (int64_t)512 +
                               rank * DVH + ch * 32;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(o + j) = make_float4(
                            __uint_as_float(ov[j]) * inv, __uint_as_float(ov[j + 1]) * inv,
                            __uint_as_float(ov[j + 2]) * inv, __uint_as_float(ov[j + 3]) * inv);
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
    e = cudaLaunchKernelEx(&cfg, hfa_tc_kernel, a);
    if (e != cudaSuccess) return e;
    return launched();
}

}  // namespace lsa
